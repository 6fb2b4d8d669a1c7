"""The allocation-free decode entry point, called through the C ABI.

mla_decode_latent_noalloc serves callers that cannot give the library device
memory at call time (an engine plugin whose enqueue must not allocate, a
latency-critical path that cannot afford cudaMalloc): it keeps the split-KV
partials in a fixed 32 MiB device array inside the library instead of a caller
workspace. It runs the same kernels on the same partition as the
workspace-based entry points (mla_decode_splitkv + mla_combine), so its
outputs must equal theirs bit for bit. The checks call it on one problem, then
on a different one (other seeds, more sequences, more partitions), then on the
first again, each time against the workspace path: the array keeps whatever the
previous call left, so a slot read before this call wrote it would show up as a
mismatch. A problem too large for the array must be refused before anything
runs. The file is named to be collected last and works both on its own and
after the other tests.
"""
import ctypes

import pytest
import torch

from mla_latent_kv_18_b200.inputs import make_inputs, to_device, workload

pytestmark = pytest.mark.gpu


def _noalloc(b, dims, q, d, num_parts, o_lat, lse):
    ckv = b.MLAPool(d["ckv_pool"].data_ptr(), d["ckv_pool"].stride(0), d["ckv_pool"].stride(1))
    kr = b.MLAPool(d["kr_pool"].data_ptr(), d["kr_pool"].stride(0), d["kr_pool"].stride(1))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return b.lib.mla_decode_latent_noalloc(
        ctypes.byref(dims), ctypes.c_void_p(q.data_ptr()), ctypes.byref(ckv), ctypes.byref(kr),
        d["ckv_pool"].shape[0], ctypes.c_void_p(d["block_table"].data_ptr()),
        d["block_table"].shape[1], ctypes.c_void_p(d["seq_lens"].data_ptr()),
        d["block_table"].shape[0], num_parts, ctypes.c_void_p(o_lat.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), stream)


def _problem(api, name, kw, seed, parts_scale):
    w = workload(name, **kw)
    d = to_device(make_inputs(w, seed=seed), "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    T = api.tile_tokens(dims)
    tiles = int(((d["seq_lens"].cpu().long() + T - 1) // T).sum())
    parts = max(1, api.num_parts_for(dims, tiles, "cuda") // parts_scale)
    q = api.absorb_q(d["q_c"], d["q_r"], d["w_uk"], dims)
    ws = api.decode_splitkv(q, d["ckv_pool"], d["kr_pool"], d["block_table"], d["seq_lens"],
                            dims, parts)
    ref_o, ref_lse = api.combine(ws, d["seq_lens"], d["block_table"].shape[1], dims, parts)
    return dict(d=d, dims=dims, q=q, parts=parts, ref_o=ref_o, ref_lse=ref_lse)


@pytest.mark.parametrize("name,kw_a,kw_b", [
    ("dsv3", dict(batch=4, seq_len=3000), dict(batch=7, seq_len=5000)),
    ("retrofit", dict(batch=6, seq_len=2000), dict(batch=11, seq_len=3100)),
])
def test_noalloc_matches_workspace_path_bitwise(name, kw_a, kw_b):
    from mla_latent_kv_18_b200 import _binding as b
    from mla_latent_kv_18_b200 import api
    # problem a uses a quarter of the default partitions, problem b the default:
    # b covers more slots of the array than a, with other values in them
    pa = _problem(api, name, kw_a, seed=21, parts_scale=4)
    pb = _problem(api, name, kw_b, seed=22, parts_scale=1)
    assert pb["parts"] > pa["parts"]
    for call, p in enumerate((pa, pb, pa)):
        o = torch.full_like(p["ref_o"], float("nan"))
        lse = torch.full_like(p["ref_lse"], float("nan"))
        assert _noalloc(b, p["dims"], p["q"], p["d"], p["parts"], o, lse) == 0
        torch.cuda.synchronize()
        assert api.get_device_error() == 0
        assert torch.equal(o, p["ref_o"]), f"o_lat differs on call {call}"
        assert torch.equal(lse, p["ref_lse"]), f"lse differs on call {call}"


def test_noalloc_refuses_problems_larger_than_its_array():
    from mla_latent_kv_18_b200 import _binding as b
    from mla_latent_kv_18_b200 import api
    dims = api.make_dims(128, 1, 128, 512, 64, 128)
    batch, parts = 256, 74      # (256 + 74) slots x 128 rows x 2 KB > 32 MiB
    assert api.workspace_bytes(dims, batch, parts) > (32 << 20)
    null = ctypes.c_void_p(0)
    pool = b.MLAPool(0, 0, 0)
    rc = b.lib.mla_decode_latent_noalloc(ctypes.byref(dims), null, ctypes.byref(pool),
                                         ctypes.byref(pool), 1, null, 1, null, batch, parts,
                                         null, null, null)
    assert rc == 1
