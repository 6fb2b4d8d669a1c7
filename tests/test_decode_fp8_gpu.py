"""Split-KV decode reading the E4M3 latent cache, against the oracle.

The GPU builds its E4M3 cache with its own quantiser (mla_append_kv_fp8) from the
seeded bf16 cache; the oracle quantises the same rows itself (the two are bit-exact,
see test_fp8_cache_gpu.py). Each c_KV element enters the products as the dequantised
bf16 value, so:
  * every (b, i, h) row of the combined result meets the decode bar against the
    oracle's attend_latent on the oracle's own dequantised cache, and
  * the result is bit-identical to the bf16 decode on that dequantised cache with the
    same partition count (same operands, same summation order).
Rows past a sequence's end in its last page (NaN codes, NaN or infinite scales, any
k_R bits) must not reach the result.
"""
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


def _check(got, ref, what):
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), what
    err = np.abs(got - ref).max()
    rel = np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30)
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max abs {err:.3e}, rel L2 {rel:.3e}"


def _token_rows(inp):
    """(seq_ids, positions, pages, slots) of every cached token, sequence-major."""
    table = inp["block_table"]
    lens = inp["seq_lens"].tolist()
    seq = torch.tensor([b for b, L in enumerate(lens) for _ in range(L)], dtype=torch.int32)
    pos = torch.tensor([t for L in lens for t in range(L)], dtype=torch.int32)
    pages = table[seq.long(), (pos // 64).long()].long()
    return seq, pos, pages, (pos % 64).long()


def _gpu_fp8_cache(api, inp, d, dims):
    """The GPU's E4M3 cache of the workload's c_KV, and its k_R pool (copied unrotated)."""
    seq, pos, pages, slots = _token_rows(inp)
    codes, scales = api.alloc_fp8_cache(inp["ckv_pool"].shape[0], inp["ckv_pool"].shape[2], "cuda")
    kr = torch.zeros_like(d["kr_pool"])
    api.append_kv_fp8(inp["ckv_pool"][pages, slots].cuda(), inp["kr_pool"][pages, slots].cuda(),
                      seq.cuda(), pos.cuda(), codes, scales, kr, d["block_table"], dims, theta=0.0)
    return codes, scales, kr


def _oracle_dequant_pool(inp):
    """The oracle's E4M3 round trip of every cached row, as a bf16 pool."""
    _, _, pages, slots = _token_rows(inp)
    codes, scales = oracle.quantize_fp8_rows(inp["ckv_pool"][pages, slots])
    pool = inp["ckv_pool"].clone()
    pool[pages, slots] = oracle.bf16_from_bits(oracle.dequant_fp8_rows(codes, scales))
    return pool


def _decode_fp8(api, d, q, codes, scales, kr, dims, parts):
    ws = api.decode_splitkv_fp8(q, codes, scales, kr, d["block_table"], d["seq_lens"], dims, parts)
    o, lse = api.combine(ws, d["seq_lens"], d["block_table"].shape[1], dims, parts)
    return o, lse


def _parts(api, dims, inp):
    lens = inp["seq_lens"].long()
    return api.num_parts_for(dims, int(((lens + 63) // 64).sum()), "cuda")


CASES = [
    # (name, workload overrides, explicit lengths, partition counts)
    ("ragged-small", dict(batch=5, ragged=(1, 1500), seq_len=0), (1, 64, 65, 700, 1500), (None, 3, 7)),
    ("dsv3", dict(), None, (None,)),
    ("ragged", dict(), None, (None, 29)),
]


@pytest.mark.parametrize("name,kw,lens,part_list", CASES, ids=[c[0] for c in CASES])
def test_decode_from_fp8_cache(api, name, kw, lens, part_list):
    base = "ragged" if name.startswith("ragged") else name
    w = workload(base, **kw)
    inp = make_inputs(w, seed=41, seq_lens=lens)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    codes, scales, kr = _gpu_fp8_cache(api, inp, d, dims)
    q = api.absorb_q(d["q_c"], d["q_r"], d["w_uk"], dims)
    pool = _oracle_dequant_pool(inp)
    pool_d = pool.cuda()
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    o_ref, lse_ref = oracle.attend_latent(q.cpu(), pool, inp["kr_pool"], inp["block_table"],
                                          inp["seq_lens"], scale)
    for parts in part_list:
        P = _parts(api, dims, inp) if parts is None else parts
        o8, lse8 = _decode_fp8(api, d, q, codes, scales, kr, dims, P)
        ws = api.decode_splitkv(q, pool_d, kr, d["block_table"], d["seq_lens"], dims, P)
        o16, lse16 = api.combine(ws, d["seq_lens"], d["block_table"].shape[1], dims, P)
        torch.cuda.synchronize()
        assert api.get_device_error() == 0
        assert torch.equal(o8, o16) and torch.equal(lse8, lse16), (name, P)
        _check(_f64(o8), o_ref, f"{name} o_lat parts={P}")
        assert np.abs(_f64(lse8) - lse_ref).max() <= 1e-3


@pytest.mark.parametrize("parts", [None, 3])
def test_decode_fp8_nonfinite_page_tails(api, parts):
    # NaN codes and NaN / infinite scales (and NaN k_R) past each sequence's end in its
    # last page leave the result bit-identical to the clean cache's
    w = workload("dsv3", batch=4, ragged=(1, 900), seq_len=0)
    inp = make_inputs(w, seed=43, seq_lens=(1, 63, 130, 900))
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    codes, scales, kr = _gpu_fp8_cache(api, inp, d, dims)
    q = api.absorb_q(d["q_c"], d["q_r"], d["w_uk"], dims)
    P = _parts(api, dims, inp) if parts is None else parts
    o_clean, lse_clean = _decode_fp8(api, d, q, codes, scales, kr, dims, P)
    specials = torch.tensor([float("nan"), float("inf"), float("-inf")], device="cuda")
    for b, L in enumerate(inp["seq_lens"].tolist()):
        used = L % 64
        if used == 0:
            continue
        page = int(inp["block_table"][b, (L - 1) // 64])
        codes[page, used:] = 0x7F                         # E4M3 NaN
        scales[page, used:] = specials[torch.arange(64 - used, device="cuda") % 3]
        kr[page, used:] = float("nan")
    o, lse = _decode_fp8(api, d, q, codes, scales, kr, dims, P)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.isfinite(o.float()).all()
    assert torch.equal(o, o_clean) and torch.equal(lse, lse_clean)


def test_decode_fp8_long_context_sampled(api):
    # the long-context shape (16 x 65536 tokens) with an E4M3 cache: bit-identical to
    # the bf16 decode on the dequantised cache, and sampled rows against the oracle
    w = workload("long")
    inp = make_inputs(w, seed=0)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    codes, scales, kr = _gpu_fp8_cache(api, inp, d, dims)
    q = api.absorb_q(d["q_c"], d["q_r"], d["w_uk"], dims)
    P = _parts(api, dims, inp)
    o8, lse8 = _decode_fp8(api, d, q, codes, scales, kr, dims, P)
    deq = api.gather_dequant_fp8(codes, scales, d["block_table"], d["seq_lens"], w.seq_len)
    pool_d = d["ckv_pool"].clone()
    t = torch.arange(w.seq_len, device="cuda")
    for b in range(w.batch):
        pool_d[d["block_table"][b, t // 64].long(), t % 64] = deq[b]
    del deq
    ws = api.decode_splitkv(q, pool_d, kr, d["block_table"], d["seq_lens"], dims, P)
    o16, lse16 = api.combine(ws, d["seq_lens"], d["block_table"].shape[1], dims, P)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(o8, o16) and torch.equal(lse8, lse16)
    # two sequences, every head, against the oracle on its own dequantised cache
    scale = oracle.default_scale(w.d_nope, w.d_rope)
    for b in (0, w.batch - 1):
        L = int(inp["seq_lens"][b])
        tt = torch.arange(L)
        pages = inp["block_table"][b, tt // 64].long()
        c, s = oracle.quantize_fp8_rows(inp["ckv_pool"][pages, tt % 64])
        pool = inp["ckv_pool"].clone()
        pool[pages, tt % 64] = oracle.bf16_from_bits(oracle.dequant_fp8_rows(c, s))
        o_ref, lse_ref = oracle.attend_latent(q[b:b + 1].cpu(), pool, inp["kr_pool"],
                                              inp["block_table"][b:b + 1], inp["seq_lens"][b:b + 1],
                                              scale)
        _check(_f64(o8[b:b + 1]), o_ref, f"long b={b}")
        assert np.abs(_f64(lse8[b:b + 1]) - lse_ref).max() <= 1e-3


@pytest.mark.parametrize("n_q", [1, 2])
def test_decode_fp8_extreme_scales_bitwise(api, n_q):
    # codes and per-token scales written directly (not through the quantiser): scales
    # from 2^-140 (products below the fp32 normal range) to 2^12 (scores ~1e8), random
    # non-NaN codes, and n_q = 2 (causal pair).
    # The decode must equal the bf16 decode on the oracle's dequantisation of the
    # same codes bit for bit: the same operands reach the same products.
    w = workload("dsv3", batch=3, heads=16, n_q=n_q, ragged=(2, 700), seq_len=0)
    inp = make_inputs(w, seed=47, seq_lens=(2, 333, 700))
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    pages = inp["ckv_pool"].shape[0]
    g = torch.Generator().manual_seed(48)
    codes = torch.randint(0, 256, (pages, 64, 512), generator=g, dtype=torch.int32).to(torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x7E                              # no NaN codes
    expo = torch.randint(-140, 13, (pages, 64), generator=g).to(torch.float32)
    scales = torch.ldexp(1.0 + torch.rand(pages, 64, generator=g), expo).to(torch.float32)
    deq = oracle.bf16_from_bits(oracle.dequant_fp8_rows(codes.numpy(), scales.numpy()))
    pool_d = deq.cuda()
    codes_d, scales_d = codes.cuda(), scales.cuda()
    q = api.absorb_q(d["q_c"], d["q_r"], d["w_uk"], dims)
    for parts in (None, 3):
        P = _parts(api, dims, inp) if parts is None else parts
        o8, lse8 = _decode_fp8(api, d, q, codes_d, scales_d, d["kr_pool"], dims, P)
        ws = api.decode_splitkv(q, pool_d, d["kr_pool"], d["block_table"], d["seq_lens"], dims, P)
        o16, lse16 = api.combine(ws, d["seq_lens"], d["block_table"].shape[1], dims, P)
        torch.cuda.synchronize()
        assert api.get_device_error() == 0
        assert torch.equal(o8, o16) and torch.equal(lse8, lse16), P
