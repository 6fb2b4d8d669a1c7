"""Cache write with the rotary embedding of k_R (mla_append_kv) against the oracle.

c_KV rows are copied bit for bit; k_R rows are the oracle's fp64 rotation within
one bf16 rounding, and bit-identical to the rotation mla_absorb_q_rope applies
to queries at the same position (keys and queries must turn alike for the
scores to depend only on relative position). Every slot not written keeps its
old bits.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_18_b200.inputs import make_inputs, to_device, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from mla_latent_kv_18_b200 import api as _api
    assert torch.cuda.is_available()
    return _api


def _f64(t):
    return t.detach().float().cpu().double().numpy()


def _bf16_rand(g, shape):
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _new_tokens(inp, n_per_seq, g):
    """n_per_seq positions per sequence (first, last, page edges and random ones)."""
    seq, pos = [], []
    for b, L in enumerate(inp["seq_lens"].tolist()):
        cand = {0, L - 1, min(63, L - 1), min(64, L - 1)}
        cand |= set(torch.randint(0, L, (n_per_seq,), generator=g).tolist())
        cand = sorted(cand)[:n_per_seq]
        seq += [b] * len(cand)
        pos += cand
    return torch.tensor(seq, dtype=torch.int32), torch.tensor(pos, dtype=torch.int32)


@pytest.mark.parametrize("name,kw", [("dsv3", dict(batch=3, heads=4, seq_len=300)),
                                     ("retrofit", dict(batch=2, heads=4, seq_len=200))])
def test_append_kv_copies_latent_and_rotates_key(api, name, kw):
    w = workload(name, **kw)
    inp = make_inputs(w, seed=21)
    d = to_device(inp, "cuda")
    g = torch.Generator().manual_seed(22)
    seq, pos = _new_tokens(inp, 12, g)
    T = seq.numel()
    ckv_new = _bf16_rand(g, (T, w.d_latent))
    kr_new = _bf16_rand(g, (T, w.d_rope))
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    ckv0, kr0 = d["ckv_pool"].clone(), d["kr_pool"].clone()
    api.append_kv(ckv_new.cuda(), kr_new.cuda(), seq.cuda(), pos.cuda(), d["ckv_pool"],
                  d["kr_pool"], d["block_table"], dims)
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    table = inp["block_table"]
    pages = torch.stack([table[b, p // 64] for b, p in zip(seq.tolist(), pos.tolist())]).long()
    slots = (pos % 64).long()
    ckv_got = d["ckv_pool"].cpu()[pages, slots]
    kr_got = d["kr_pool"].cpu()[pages, slots]
    assert torch.equal(ckv_got, ckv_new)
    ref = oracle.rope(kr_new.reshape(T, 1, w.d_rope), pos.numpy()).reshape(T, w.d_rope)
    err = np.abs(_f64(kr_got) - ref) / (2.0 ** -7 * np.abs(ref) + 1e-3)
    assert err.max() <= 1.0, err.max()
    # the queries' rotation (absorb-in with RoPE, one head, zero latent part) is bit-identical
    dims1 = api.make_dims(1, 1, w.d_nope, w.d_latent, w.d_rope, w.d_v)
    q_c = torch.zeros(T, 1, 1, w.d_nope, dtype=torch.bfloat16, device="cuda")
    w_uk = torch.zeros(1, w.d_nope, w.d_latent, dtype=torch.bfloat16, device="cuda")
    q = api.absorb_q_rope(q_c, kr_new.reshape(T, 1, 1, w.d_rope).cuda(), w_uk, dims1, pos.cuda())
    torch.cuda.synchronize()
    assert torch.equal(q[:, 0, 0, w.d_latent:].cpu(), kr_got)
    # nothing else moved
    mask = torch.ones(ckv0.shape[:2], dtype=torch.bool)
    mask[pages, slots] = False
    assert torch.equal(d["ckv_pool"].cpu()[mask], ckv0.cpu()[mask])
    assert torch.equal(d["kr_pool"].cpu()[mask], kr0.cpu()[mask])
    # theta <= 0: k_R copied unrotated
    api.append_kv(ckv_new.cuda(), kr_new.cuda(), seq.cuda(), pos.cuda(), d["ckv_pool"],
                  d["kr_pool"], d["block_table"], dims, theta=0.0)
    torch.cuda.synchronize()
    assert torch.equal(d["kr_pool"].cpu()[pages, slots], kr_new)


def test_cache_built_by_appends_decodes_with_relative_rope(api):
    # write every token of every sequence through mla_append_kv (rotating k_R at its
    # position), rotate the query with mla_absorb_q_rope at its position, decode, and
    # compare with the oracle fed the same rotations computed in fp64
    w = workload("dsv3", batch=2, heads=16, seq_len=400)
    inp = make_inputs(w, seed=23)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    table = inp["block_table"]
    lens = inp["seq_lens"].tolist()
    seq = torch.tensor([b for b, L in enumerate(lens) for _ in range(L)], dtype=torch.int32)
    pos = torch.tensor([t for L in lens for t in range(L)], dtype=torch.int32)
    pages = torch.stack([table[b, p // 64] for b, p in zip(seq.tolist(), pos.tolist())]).long()
    slots = (pos % 64).long()
    ckv_new = inp["ckv_pool"][pages, slots]            # the workload's latents, token order
    kr_raw = inp["kr_pool"][pages, slots]              # read as unrotated keys
    ckv_pool = torch.zeros_like(d["ckv_pool"])
    kr_pool = torch.zeros_like(d["kr_pool"])
    api.append_kv(ckv_new.cuda(), kr_raw.cuda(), seq.cuda(), pos.cuda(), ckv_pool, kr_pool,
                  d["block_table"], dims)
    qpos = torch.tensor([L - 1 for L in lens], dtype=torch.int32)
    q = api.absorb_q_rope(d["q_c"], d["q_r"], d["w_uk"], dims, qpos.cuda())
    parts = api.num_parts_for(dims, sum((L + 63) // 64 for L in lens), "cuda")
    ws = api.decode_splitkv(q, ckv_pool, kr_pool, d["block_table"], d["seq_lens"], dims, parts)
    out = api.combine_absorb_out(ws, d["seq_lens"], table.shape[1], dims, parts, d["w_uv"])
    torch.cuda.synchronize()
    assert api.get_device_error() == 0
    assert torch.equal(ckv_pool.cpu()[pages, slots], ckv_new)
    # oracle inputs: fp64 rotations rounded to bf16 once (the cache and Q hold bf16)
    kr_rot = oracle.rope(kr_raw.reshape(-1, 1, w.d_rope), pos.numpy()).reshape(-1, w.d_rope)
    qr_rot = oracle.rope(inp["q_r"].reshape(w.batch, w.heads, w.d_rope), qpos.numpy())
    ref_inp = dict(inp)
    kr_ref = inp["kr_pool"].clone()
    kr_ref[pages, slots] = torch.tensor(kr_rot, dtype=torch.float32).to(torch.bfloat16)
    ref_inp["kr_pool"] = kr_ref
    ref_inp["q_r"] = torch.tensor(qr_rot, dtype=torch.float32).to(torch.bfloat16).reshape(
        inp["q_r"].shape)
    args = [ref_inp[k] for k in ("q_c", "q_r", "ckv_pool", "kr_pool", "block_table", "seq_lens",
                                 "w_uk", "w_uv")]
    ref = oracle.decode_decompress(*args)
    got = _f64(out)
    err = np.abs(got - ref).max()
    rel = np.linalg.norm((got - ref).ravel()) / np.linalg.norm(ref.ravel())
    assert err <= 1e-2 and rel <= 5e-3, (err, rel)


def test_append_kv_bad_position_sets_bounds_error(api):
    w = workload("dsv3", batch=2, heads=4, seq_len=100)
    inp = make_inputs(w, seed=24)
    d = to_device(inp, "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    g = torch.Generator().manual_seed(25)
    ckv_new = _bf16_rand(g, (3, w.d_latent)).cuda()
    kr_new = _bf16_rand(g, (3, w.d_rope)).cuda()
    seq = torch.tensor([0, 1, 5], dtype=torch.int32, device="cuda")          # sequence 5: none
    pos = torch.tensor([10, 128 * 64, 3], dtype=torch.int32, device="cuda")   # past the table
    api.append_kv(ckv_new, kr_new, seq, pos, d["ckv_pool"], d["kr_pool"], d["block_table"], dims)
    torch.cuda.synchronize()
    assert api.get_device_error() == 4
    page = int(inp["block_table"][0, 0])
    assert torch.equal(d["ckv_pool"][page, 10].cpu(), ckv_new[0].cpu())      # the valid one landed
    assert api.get_device_error() == 0
