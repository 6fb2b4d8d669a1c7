"""The allocation-free decode entry point, called through the C ABI.

mla_decode_latent_noalloc serves callers that cannot give the library device
memory at call time (an engine plugin whose enqueue must not allocate, a
latency-critical path that cannot afford cudaMalloc): it keeps the split-KV
partials in a fixed 32 MiB device array inside the library instead of a caller
workspace. These checks compare it with the workspace-based entry points
(mla_decode_splitkv + mla_combine) on the same inputs, twice in a row (the
array keeps the previous call's contents), and check that a problem too large
for the array is refused before anything runs. The file is named to be
collected last and works both on its own and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from mla_latent_kv_18_b200.inputs import make_inputs, to_device, workload

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 1e-2, 5e-3


def _close(got, ref, what):
    got = got.float().cpu().double().numpy()
    ref = ref.float().cpu().double().numpy()
    assert np.isfinite(got).all(), what
    err = np.abs(got - ref).max()
    rel = np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30)
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max abs {err:.3e}, rel L2 {rel:.3e}"


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


@pytest.mark.parametrize("name,kw", [("dsv3", dict(batch=4, seq_len=3000)),
                                     ("retrofit", dict(batch=6, seq_len=2000))])
def test_noalloc_matches_workspace_path_twice(name, kw):
    from mla_latent_kv_18_b200 import _binding as b
    from mla_latent_kv_18_b200 import api
    w = workload(name, **kw)
    d = to_device(make_inputs(w, seed=21), "cuda")
    dims = api.dims_for(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"])
    T = api.tile_tokens(dims)
    tiles = int(((d["seq_lens"].cpu().long() + T - 1) // T).sum())
    parts = api.num_parts_for(dims, tiles, "cuda")
    q = api.absorb_q(d["q_c"], d["q_r"], d["w_uk"], dims)
    ws = api.decode_splitkv(q, d["ckv_pool"], d["kr_pool"], d["block_table"], d["seq_lens"],
                            dims, parts)
    ref_o, ref_lse = api.combine(ws, d["seq_lens"], d["block_table"].shape[1], dims, parts)
    for call in range(2):
        o = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _noalloc(b, dims, q, d, parts, o, lse) == 0
        torch.cuda.synchronize()
        assert api.get_device_error() == 0
        _close(o, ref_o, f"o_lat call {call}")
        _close(lse, ref_lse, f"lse call {call}")


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
