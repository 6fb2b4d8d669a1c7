"""The E4M3 latent cache on the GPU against the oracle.

Quantisation on cache write (codes and per-token scales) and the dequantising
gather are integer/byte work with every floating-point decision taken in IEEE
fp32 on both sides, so both are checked bit for bit. The decompress branch read
from the E4M3 cache equals the bf16 branch on the dequantised cache bit for bit,
and meets the prefill output bar against the oracle run on the oracle's own
dequantised cache. The GPU side builds its E4M3 cache with its own quantiser
(mla_append_kv_fp8) from the seeded bf16 cache; the oracle quantises the same
bf16 rows itself.
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


def _token_rows(inp):
    """(seq_ids, positions, pages, slots) of every cached token, sequence-major."""
    table = inp["block_table"]
    lens = inp["seq_lens"].tolist()
    seq = torch.tensor([b for b, L in enumerate(lens) for _ in range(L)], dtype=torch.int32)
    pos = torch.tensor([t for L in lens for t in range(L)], dtype=torch.int32)
    pages = table[seq.long(), (pos // 64).long()].long()
    return seq, pos, pages, (pos % 64).long()


def _gpu_fp8_cache(api, inp, d, dims):
    """The GPU's E4M3 cache of the workload's bf16 c_KV (k_R copied unrotated)."""
    seq, pos, pages, slots = _token_rows(inp)
    codes, scales = api.alloc_fp8_cache(inp["ckv_pool"].shape[0], inp["ckv_pool"].shape[2], "cuda")
    kr = torch.zeros_like(d["kr_pool"])
    api.append_kv_fp8(inp["ckv_pool"][pages, slots].cuda(), inp["kr_pool"][pages, slots].cuda(),
                      seq.cuda(), pos.cuda(), codes, scales, kr, d["block_table"], dims, theta=0.0)
    return codes, scales, kr


def _oracle_dequant_pool(inp):
    """The oracle's E4M3 round trip of every cached row, as a bf16 pool."""
    _, _, pages, slots = _token_rows(inp)
    rows = inp["ckv_pool"][pages, slots]
    codes, scales = oracle.quantize_fp8_rows(rows)
    pool = inp["ckv_pool"].clone()
    pool[pages, slots] = oracle.bf16_from_bits(oracle.dequant_fp8_rows(codes, scales))
    return pool, codes, scales


@pytest.mark.parametrize("name,kw", [("dsv3", dict(batch=3, heads=4, ragged=(70, 300), seq_len=0)),
                                     ("retrofit", dict(batch=2, heads=4, seq_len=150))])
def test_append_fp8_codes_and_scales_are_bit_exact(api, name, kw):
    w = workload(name, **kw)
    inp = make_inputs(w, seed=31)
    # rows of very different magnitudes, and an all-zero row
    _, _, pages, slots = _token_rows(inp)
    g = torch.Generator().manual_seed(32)
    mag = torch.exp2(torch.randint(-12, 10, (inp["ckv_pool"].shape[0], 64, 1), generator=g).float())
    inp["ckv_pool"] = (inp["ckv_pool"].float() * mag).to(torch.bfloat16)
    inp["ckv_pool"][pages[5], slots[5]] = 0
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    codes, scales, kr = _gpu_fp8_cache(api, inp, d, dims)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    want_codes, want_scales = oracle.quantize_fp8_rows(inp["ckv_pool"][pages, slots])
    np.testing.assert_array_equal(codes.cpu()[pages, slots].numpy(), want_codes)
    np.testing.assert_array_equal(scales.cpu()[pages, slots].numpy(), want_scales)
    assert torch.equal(kr.cpu()[pages, slots], inp["kr_pool"][pages, slots])


@pytest.mark.parametrize("name,kw", [("dsv3", dict(batch=4, heads=4, ragged=(1, 700), seq_len=0)),
                                     ("retrofit", dict(batch=3, heads=4, seq_len=200))])
def test_dequantising_gather_is_bit_exact(api, name, kw):
    w = workload(name, **kw)
    inp = make_inputs(w, seed=33, seq_lens=(1, 64, 65, 700)[:w.batch] if name == "dsv3" else None)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    codes, scales, _ = _gpu_fp8_cache(api, inp, d, dims)
    max_len = int(inp["seq_lens"].max()) + 3
    sentinel = torch.full((w.batch, max_len, w.d_latent), 7.0, dtype=torch.bfloat16, device="cuda")
    out = api.gather_dequant_fp8(codes, scales, d["block_table"], d["seq_lens"], max_len,
                                 out=sentinel)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    pool, _, _ = _oracle_dequant_pool(inp)
    for b, L in enumerate(inp["seq_lens"].tolist()):
        t = torch.arange(L)
        want = pool[inp["block_table"][b, t // 64].long(), t % 64]
        assert torch.equal(out[b, :L].cpu(), want)
        assert (out[b, L:] == 7.0).all()                  # rows past the end untouched


@pytest.mark.parametrize("M,lens", [(256, (256, 700)), (130, (300, 130))])
def test_prefill_from_fp8_cache(api, M, lens):
    w = workload("prefill", batch=len(lens), n_q=M, heads=4, seq_len=0,
                 ragged=(min(lens), max(lens)))
    inp = make_inputs(w, seed=M, seq_lens=lens)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    codes, scales, _ = _gpu_fp8_cache(api, inp, d, dims)
    ws8 = api.decompress_kv_fp8(codes, scales, d["block_table"], d["seq_lens"], d["w_uk"],
                                d["w_uv"], dims)
    out, lse = api.prefill_attention(d["q_c"], d["q_r"], d["kr_pool"], d["block_table"],
                                     d["seq_lens"], dims, ws8)
    # the bf16 branch on the GPU's own dequantised cache: identical bits
    _, _, pages, slots = _token_rows(inp)
    deq = api.gather_dequant_fp8(codes, scales, d["block_table"], d["seq_lens"],
                                 int(max(lens)))
    bpool = d["ckv_pool"].clone()
    seq, pos, _, _ = _token_rows(inp)
    bpool[pages.cuda(), slots.cuda()] = deq[seq.long().cuda(), pos.long().cuda()]
    ws16 = api.decompress_kv(bpool, d["block_table"], d["seq_lens"], d["w_uk"], d["w_uv"], dims)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    B, max_pages = d["block_table"].shape
    k8, v8 = api.prefill_workspace_views(ws8, dims, B, max_pages)
    k16, v16 = api.prefill_workspace_views(ws16, dims, B, max_pages)
    for b, L in enumerate(lens):                     # the rows the decompression writes
        n = (L + 127) // 128 * 128
        assert torch.equal(k8[b, :, :n], k16[b, :, :n]) and torch.equal(v8[b, :, :n], v16[b, :, :n])
    # against the oracle on the oracle's dequantised cache
    pool, _, _ = _oracle_dequant_pool(inp)
    ref_inp = dict(inp, ckv_pool=pool)
    args = [ref_inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                                 "w_uk", "w_uv")]
    ref, lse_ref = oracle.prefill_decompress(*args)
    got = _f64(out)
    vis = np.array([[L - M + i + 1 for i in range(M)] for L in lens])
    many = vis >= 64
    err = np.abs(got[many] - ref[many]).max()
    rel = np.linalg.norm((got - ref).ravel()) / np.linalg.norm(ref.ravel())
    worst = (np.abs(got - ref) / (MAX_ABS + 2.0 ** -7 * np.abs(ref))).max()
    assert err <= MAX_ABS and rel <= REL_L2 and worst <= 1.0, (err, rel, worst)
    assert np.abs(_f64(lse) - lse_ref).max() <= LSE_ABS


def test_dequantising_gather_full_size_sampled(api):
    # the long-context cache (16 x 65536 tokens): quantised on write, gathered back, and
    # checked bit for bit on sampled rows against the oracle's round trip
    w = workload("long")
    inp = make_inputs(w, seed=0)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    codes, scales, _ = _gpu_fp8_cache(api, inp, d, dims)
    out = api.gather_dequant_fp8(codes, scales, d["block_table"], d["seq_lens"], w.seq_len)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    rng = np.random.default_rng(0)
    b = torch.from_numpy(rng.integers(0, w.batch, 512))
    t = torch.from_numpy(rng.integers(0, w.seq_len, 512))
    rows = inp["ckv_pool"][inp["block_table"][b, t // 64].long(), t % 64]
    c, s = oracle.quantize_fp8_rows(rows)
    want = oracle.bf16_from_bits(oracle.dequant_fp8_rows(c, s))
    assert torch.equal(out[b.cuda(), t.cuda()].cpu(), want)
