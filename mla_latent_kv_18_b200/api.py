"""Python API over the C ABI: MLA decode with matrix absorption on a paged
latent cache. PyTorch supplies device memory and the current stream only;
every step runs in the library's sm_100a kernels.

    q   = absorb_q(q_c, q_r, w_uk)                         # [B, n_q, H, d_c + d_R]
    ws, parts = decode_splitkv(q, ckv_pool, kr_pool, block_table, seq_lens)
    o, lse = combine(ws, seq_lens, parts, ...)             # [B, n_q, H, d_c]
    out = absorb_out(o, w_uv)                              # [B, n_q, H, d_v]

or ``decode(...)`` for all four. A step with many query tokens per sequence
(``prefill``) decompresses the cache per head instead; ``attend`` routes a
step by its query count.
"""
import ctypes

import torch

from . import _binding as _b

_NUM_SMS = {}


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _num_sms(device):
    idx = torch.device(device).index
    if idx is None:
        idx = torch.cuda.current_device()
    if idx not in _NUM_SMS:
        _NUM_SMS[idx] = torch.cuda.get_device_properties(idx).multi_processor_count
    return _NUM_SMS[idx]


def make_dims(heads, n_q, d_nope, d_latent, d_rope, d_v, page_size=64, scale=0.0):
    return _b.MLADims(heads, n_q, d_nope, d_latent, d_rope, d_v, page_size, float(scale))


def dims_for(q_c, q_r, w_uk, w_uv, page_size=64, scale=0.0):
    """Dims from tensor shapes: q_c [B, n_q, H, d_n], q_r [.., d_R], w_uk [H, d_n, d_c],
    w_uv [H, d_c, d_v]."""
    H, d_n, d_c = w_uk.shape
    return make_dims(H, q_c.shape[1], d_n, d_c, q_r.shape[-1], w_uv.shape[-1], page_size, scale)


def _pool(t):
    """A [pages, 64, C] (possibly channel-sliced) bf16 view -> mla_pool."""
    assert t.dtype == torch.bfloat16 and t.dim() == 3 and t.stride(2) == 1
    return _b.MLAPool(t.data_ptr(), t.stride(0), t.stride(1))


def absorb_q(q_c, q_r, w_uk, dims, out=None, stream=None):
    T = q_c.numel() // (dims.num_heads * dims.d_nope)
    if out is None:
        out = torch.empty(q_c.shape[:-1] + (dims.d_latent + dims.d_rope,), dtype=torch.bfloat16,
                          device=q_c.device)
    _b.check(_b.lib.mla_absorb_q(ctypes.byref(dims), _ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(out),
                                 T, _stream(stream)), "mla_absorb_q")
    return out


def num_parts_for(dims, total_tiles, device=None):
    return _b.lib.mla_decode_num_parts(ctypes.byref(dims), int(total_tiles),
                                       _num_sms(device or torch.cuda.current_device()))


def tile_tokens(dims):
    return 64 if dims.d_latent == 512 else 128


def workspace_bytes(dims, batch, num_parts):
    return _b.lib.mla_decode_workspace_bytes(ctypes.byref(dims), batch, num_parts)


def alloc_workspace(dims, batch, num_parts, device):
    nbytes = workspace_bytes(dims, batch, num_parts)
    if nbytes == 0:
        raise _b.MLAError(1, "mla_decode_workspace_bytes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def workspace_views(ws, dims, batch, num_parts):
    """(o_part [slots, R, d_c] fp32, lse_part [slots, R] fp32) views of a workspace."""
    slots = batch + num_parts
    R = dims.n_q * dims.num_heads
    o_bytes = (slots * R * dims.d_latent * 4 + 255) // 256 * 256
    o = ws[:slots * R * dims.d_latent * 4].view(torch.float32).view(slots, R, dims.d_latent)
    lse = ws[o_bytes:o_bytes + slots * R * 4].view(torch.float32).view(slots, R)
    return o, lse


def plan(dims, seq_lens_host, max_pages, num_parts):
    """Host replica of the kernels' partition plan: (part_first, slot_count, slot_base, slots)."""
    lens = torch.as_tensor(seq_lens_host, dtype=torch.int32).contiguous()
    B = lens.numel()
    pf = torch.empty(B, dtype=torch.int32)
    cnt = torch.empty(B, dtype=torch.int32)
    base = torch.empty(B, dtype=torch.int64)
    total = _b.lib.mla_decode_plan(ctypes.byref(dims), _ptr(lens), max_pages, B, num_parts,
                                   _ptr(pf), _ptr(cnt), _ptr(base))
    if total < 0:
        raise _b.MLAError(1, "mla_decode_plan")
    return pf, cnt, base, total


def decode_splitkv(q, ckv_pool, kr_pool, block_table, seq_lens, dims, num_parts,
                   workspace=None, stream=None):
    B = block_table.shape[0]
    if workspace is None:
        workspace = alloc_workspace(dims, B, num_parts, q.device)
    ckv, kr = _pool(ckv_pool), _pool(kr_pool)
    _b.check(_b.lib.mla_decode_splitkv(ctypes.byref(dims), _ptr(q), ctypes.byref(ckv),
                                       ctypes.byref(kr), ckv_pool.shape[0], _ptr(block_table),
                                       block_table.shape[1], _ptr(seq_lens), B, num_parts,
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
             "mla_decode_splitkv")
    return workspace


def decode_splitkv_fp8(q, ckv8_pool, scales, kr_pool, block_table, seq_lens, dims, num_parts,
                       workspace=None, stream=None):
    """decode_splitkv reading the E4M3 cache (codes [pages, 64, 512] uint8, scales
    [pages, 64] fp32, k_R bf16); combine() reads the workspace as usual."""
    B = block_table.shape[0]
    if workspace is None:
        workspace = alloc_workspace(dims, B, num_parts, q.device)
    assert scales.dtype == torch.float32 and scales.is_contiguous()
    _b.check(_b.lib.mla_decode_splitkv_fp8(ctypes.byref(dims), _ptr(q),
                                           ctypes.byref(_pool8(ckv8_pool)), _ptr(scales),
                                           ctypes.byref(_pool(kr_pool)), ckv8_pool.shape[0],
                                           _ptr(block_table), block_table.shape[1], _ptr(seq_lens),
                                           B, num_parts, _ptr(workspace), workspace.numel(),
                                           _stream(stream)),
             "mla_decode_splitkv_fp8")
    return workspace


def combine(workspace, seq_lens, max_pages, dims, num_parts, o_lat=None, lse_out=None,
            with_lse=True, stream=None):
    B = seq_lens.shape[0]
    R = dims.n_q * dims.num_heads
    dev = workspace.device
    if o_lat is None:
        o_lat = torch.empty(B, dims.n_q, dims.num_heads, dims.d_latent, dtype=torch.bfloat16,
                            device=dev)
    if with_lse and lse_out is None:
        lse_out = torch.empty(B, dims.n_q, dims.num_heads, dtype=torch.float32, device=dev)
    _b.check(_b.lib.mla_combine(ctypes.byref(dims), _ptr(workspace), workspace.numel(),
                                _ptr(seq_lens), max_pages, B, num_parts, _ptr(o_lat),
                                _ptr(lse_out) if with_lse else None, _stream(stream)),
             "mla_combine")
    return o_lat, lse_out


def absorb_q_rope(q_c, q_r, w_uk, dims, positions, theta=10000.0, out=None, stream=None):
    """absorb_q with q_r rotated by the rotary embedding at positions [T] (int32, device)."""
    T = q_c.numel() // (dims.num_heads * dims.d_nope)
    if out is None:
        out = torch.empty(q_c.shape[:-1] + (dims.d_latent + dims.d_rope,), dtype=torch.bfloat16,
                          device=q_c.device)
    assert positions.dtype == torch.int32 and positions.numel() == T
    _b.check(_b.lib.mla_absorb_q_rope(ctypes.byref(dims), _ptr(q_c), _ptr(q_r), _ptr(w_uk),
                                      _ptr(positions), float(theta), _ptr(out), T, _stream(stream)),
             "mla_absorb_q_rope")
    return out


def absorb_out(o_lat, w_uv, dims, out=None, stream=None):
    T = o_lat.numel() // (dims.num_heads * dims.d_latent)
    if out is None:
        out = torch.empty(o_lat.shape[:-1] + (dims.d_v,), dtype=torch.bfloat16, device=o_lat.device)
    _b.check(_b.lib.mla_absorb_out(ctypes.byref(dims), _ptr(o_lat), _ptr(w_uv), _ptr(out), T,
                                   _stream(stream)), "mla_absorb_out")
    return out


def append_kv(ckv_new, kr_new, seq_ids, positions, ckv_pool, kr_pool, block_table, dims,
              theta=10000.0, stream=None):
    """Write new tokens' c_KV and RoPE-rotated k_R into the paged pools (in place).
    ckv_new [T, d_c], kr_new [T, d_R] (unrotated) bf16; seq_ids, positions [T] int32.
    theta <= 0 copies k_R unrotated."""
    T = ckv_new.shape[0]
    B, max_pages = block_table.shape
    _b.check(_b.lib.mla_append_kv(ctypes.byref(dims), _ptr(ckv_new), _ptr(kr_new), _ptr(seq_ids),
                                  _ptr(positions), T, float(theta), ctypes.byref(_pool(ckv_pool)),
                                  ctypes.byref(_pool(kr_pool)), ckv_pool.shape[0],
                                  _ptr(block_table), max_pages, B, _stream(stream)),
             "mla_append_kv")


def _pool8(t):
    """A [pages, 64, C] uint8 E4M3 code pool -> mla_pool (strides in bytes)."""
    assert t.dtype == torch.uint8 and t.dim() == 3 and t.stride(2) == 1
    return _b.MLAPool(t.data_ptr(), t.stride(0), t.stride(1))


def alloc_fp8_cache(num_pages, d_latent, device):
    """(codes [pages, 64, d_latent] uint8, scales [pages, 64] float32), zeroed."""
    return (torch.zeros(num_pages, 64, d_latent, dtype=torch.uint8, device=device),
            torch.zeros(num_pages, 64, dtype=torch.float32, device=device))


def append_kv_fp8(ckv_new, kr_new, seq_ids, positions, ckv8_pool, scales, kr_pool, block_table,
                  dims, theta=10000.0, stream=None):
    """As append_kv, quantising c_KV into the E4M3 cache (codes + per-token scales)."""
    T = ckv_new.shape[0]
    B, max_pages = block_table.shape
    _b.check(_b.lib.mla_append_kv_fp8(ctypes.byref(dims), _ptr(ckv_new), _ptr(kr_new),
                                      _ptr(seq_ids), _ptr(positions), T, float(theta),
                                      ctypes.byref(_pool8(ckv8_pool)), _ptr(scales),
                                      ctypes.byref(_pool(kr_pool)), ckv8_pool.shape[0],
                                      _ptr(block_table), max_pages, B, _stream(stream)),
             "mla_append_kv_fp8")


def gather_dequant_fp8(ckv8_pool, scales, block_table, seq_lens, max_len, out=None, stream=None):
    """Dense bf16 [B, max_len, d_latent] of the dequantised cache rows (others untouched)."""
    B, max_pages = block_table.shape
    width = ckv8_pool.shape[2]
    if out is None:
        out = torch.zeros(B, max_len, width, dtype=torch.bfloat16, device=ckv8_pool.device)
    _b.check(_b.lib.mla_gather_dequant_fp8(ctypes.byref(_pool8(ckv8_pool)), _ptr(scales), width,
                                           ckv8_pool.shape[0], _ptr(block_table), max_pages,
                                           _ptr(seq_lens), B, max_len, _ptr(out), _stream(stream)),
             "mla_gather_dequant_fp8")
    return out


def decompress_kv_fp8(ckv8_pool, scales, block_table, seq_lens, w_uk, w_uv, dims, workspace=None,
                      stream=None):
    """decompress_kv reading the E4M3 cache."""
    B, max_pages = block_table.shape
    if workspace is None:
        workspace = alloc_prefill_workspace(dims, B, max_pages, ckv8_pool.device)
    _b.check(_b.lib.mla_decompress_kv_fp8(ctypes.byref(dims), ctypes.byref(_pool8(ckv8_pool)),
                                          _ptr(scales), ckv8_pool.shape[0], _ptr(block_table),
                                          max_pages, _ptr(seq_lens), B, _ptr(w_uk), _ptr(w_uv),
                                          _ptr(workspace), workspace.numel(), _stream(stream)),
             "mla_decompress_kv_fp8")
    return workspace


def get_device_error(stream=None):
    code = ctypes.c_int32(0)
    _b.check(_b.lib.mla_get_device_error(ctypes.byref(code), _stream(stream)),
             "mla_get_device_error")
    return code.value


def combine_absorb_out(workspace, seq_lens, max_pages, dims, num_parts, w_uv, out=None,
                       lse_out=None, stream=None):
    """Combine and absorb-out in one call: out [B, n_q, H, d_v] bf16."""
    B = seq_lens.shape[0]
    if out is None:
        out = torch.empty((B, dims.n_q, dims.num_heads, dims.d_v), dtype=torch.bfloat16,
                          device=workspace.device)
    _b.check(_b.lib.mla_combine_absorb_out(ctypes.byref(dims), _ptr(workspace), workspace.numel(),
                                           _ptr(seq_lens), max_pages, B, num_parts, _ptr(w_uv),
                                           _ptr(out), _ptr(lse_out), _stream(stream)),
             "mla_combine_absorb_out")
    return out


def debug_gather(pool, block_table, seq_lens, max_len, out=None, stream=None):
    """Gathered rows of a [pages, 64, width] (possibly channel-sliced) pool:
    out[b, t, :] = pool[block_table[b, t // 64], t % 64, :] for t < seq_lens[b]
    (bf16 bit copy; other rows of out are left as they were, zeros if allocated
    here). Uses the decode calls' page lookup and TMA pool descriptors."""
    B, max_pages = block_table.shape
    width = pool.shape[2]
    if out is None:
        out = torch.zeros((B, max_len, width), dtype=torch.bfloat16, device=pool.device)
    p = _pool(pool)
    _b.check(_b.lib.mla_debug_gather(ctypes.byref(p), width, pool.shape[0], _ptr(block_table),
                                     max_pages, _ptr(seq_lens), B, max_len, _ptr(out),
                                     _stream(stream)),
             "mla_debug_gather")
    return out


def debug_wait_timeout(timeout_ns, stream=None):
    _b.check(_b.lib.mla_debug_wait_timeout(int(timeout_ns), _stream(stream)),
             "mla_debug_wait_timeout")


class Decoder:
    """All four steps with fixed shapes; buffers allocated once (by PyTorch).

    total_tiles: sum over sequences of ceil(L_b / tile_tokens) -- decides the
    number of partitions; pass the host-side value when known.
    """

    def __init__(self, dims, batch, max_pages, total_tiles, device):
        self.dims = dims
        self.batch = batch
        self.max_pages = max_pages
        self.num_parts = num_parts_for(dims, total_tiles, device)
        self.workspace = alloc_workspace(dims, batch, self.num_parts, device)
        H, n_q = dims.num_heads, dims.n_q
        self.q = torch.empty(batch, n_q, H, dims.d_latent + dims.d_rope, dtype=torch.bfloat16,
                             device=device)
        self.o_lat = torch.empty(batch, n_q, H, dims.d_latent, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(batch, n_q, H, dtype=torch.float32, device=device)
        self.out = torch.empty(batch, n_q, H, dims.d_v, dtype=torch.bfloat16, device=device)

    def __call__(self, q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv,
                 stream=None):
        absorb_q(q_c, q_r, w_uk, self.dims, out=self.q, stream=stream)
        decode_splitkv(self.q, ckv_pool, kr_pool, block_table, seq_lens, self.dims, self.num_parts,
                       workspace=self.workspace, stream=stream)
        combine(self.workspace, seq_lens, self.max_pages, self.dims, self.num_parts,
                o_lat=self.o_lat, lse_out=self.lse, stream=stream)
        absorb_out(self.o_lat, w_uv, self.dims, out=self.out, stream=stream)
        return self.out


# (partition count, workspace) per (dims, batch, table width, tile total, device,
# stream): decode() plans and allocates its workspace once per shape.
_DECODE_PLANS = {}


def _decode_plan(dims, batch, max_pages, total_tiles, device, stream):
    key = (tuple(getattr(dims, f) for f, _ in dims._fields_), batch, max_pages, total_tiles,
           torch.device(device), stream.cuda_stream)
    plan = _DECODE_PLANS.get(key)
    if plan is None:
        parts = num_parts_for(dims, total_tiles, device)
        plan = (parts, alloc_workspace(dims, batch, parts, device))
        _DECODE_PLANS[key] = plan
    return plan


def decode(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv, total_tiles=None,
           scale=0.0, stream=None):
    """One decode step. Returns (out [B,n_q,H,d_v], o_lat [B,n_q,H,d_c], lse [B,n_q,H]).

    Serving-shaped: nothing is read back from the device. The partition count
    comes from total_tiles when given (sum over sequences of ceil(L_b / tile)),
    else from the block table's capacity (every sequence at max_pages pages);
    the plan and the split-KV workspace are made once per (shape, stream) and
    reused, and outputs come from PyTorch's caching allocator, so a warm call
    does not allocate device memory. Calls on one stream reuse its workspace in
    order; calls on different streams get different workspaces."""
    dims = dims_for(q_c, q_r, w_uk, w_uv, ckv_pool.shape[1], scale)
    B, max_pages = block_table.shape
    s = stream if stream is not None else torch.cuda.current_stream(q_c.device)
    if total_tiles is None:
        T = tile_tokens(dims)
        total_tiles = B * ((max_pages * dims.page_size + T - 1) // T)
    parts, ws = _decode_plan(dims, B, max_pages, int(total_tiles), q_c.device, s)
    q = absorb_q(q_c, q_r, w_uk, dims, stream=s)
    decode_splitkv(q, ckv_pool, kr_pool, block_table, seq_lens, dims, parts, workspace=ws, stream=s)
    o_lat, lse = combine(ws, seq_lens, max_pages, dims, parts, stream=s)
    out = absorb_out(o_lat, w_uv, dims, stream=s)
    return out, o_lat, lse


# ----------------------------------------------------------------------------
# prefill through the decompress branch
# ----------------------------------------------------------------------------

PREFILL_THRESHOLD = 256   # query tokens per sequence from which the decompress branch is taken


def prefill_workspace_bytes(dims, batch, max_pages):
    n = _b.lib.mla_prefill_workspace_bytes(ctypes.byref(dims), batch, max_pages)
    if n == 0:
        raise _b.MLAError(2, "mla_prefill_workspace_bytes")
    return n


def alloc_prefill_workspace(dims, batch, max_pages, device):
    return torch.empty(prefill_workspace_bytes(dims, batch, max_pages), dtype=torch.uint8,
                       device=device)


def prefill_workspace_views(ws, dims, batch, max_pages):
    """(K_nope, V) views [B, H, Lpad, 128] of a prefill workspace."""
    l_pad = (max_pages * 64 + 127) // 128 * 128
    n = batch * dims.num_heads * l_pad * 128
    half = (n * 2 + 255) // 256 * 256
    k = ws[:n * 2].view(torch.bfloat16).view(batch, dims.num_heads, l_pad, 128)
    v = ws[half:half + n * 2].view(torch.bfloat16).view(batch, dims.num_heads, l_pad, 128)
    return k, v


def decompress_kv(ckv_pool, block_table, seq_lens, w_uk, w_uv, dims, workspace=None,
                  stream=None):
    """K_nope = c_KV W_UK^T and V = c_KV W_UV per head into the prefill workspace."""
    B, max_pages = block_table.shape
    if workspace is None:
        workspace = alloc_prefill_workspace(dims, B, max_pages, ckv_pool.device)
    _b.check(_b.lib.mla_decompress_kv(ctypes.byref(dims), ctypes.byref(_pool(ckv_pool)),
                                      ckv_pool.shape[0], _ptr(block_table), max_pages,
                                      _ptr(seq_lens), B, _ptr(w_uk), _ptr(w_uv), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "mla_decompress_kv")
    return workspace


def prefill_attention(q_c, q_r, kr_pool, block_table, seq_lens, dims, workspace, out=None,
                      lse=None, stream=None):
    """Causal attention of the M = q_c.shape[1] last tokens of each sequence over the
    decompressed cache. Returns (out [B, M, H, 128], lse [B, M, H])."""
    B, max_pages = block_table.shape
    M, H = q_c.shape[1], dims.num_heads
    if out is None:
        out = torch.empty(B, M, H, dims.d_v, dtype=torch.bfloat16, device=q_c.device)
    if lse is None:
        lse = torch.empty(B, M, H, dtype=torch.float32, device=q_c.device)
    _b.check(_b.lib.mla_prefill_attention(ctypes.byref(dims), _ptr(q_c), _ptr(q_r),
                                          ctypes.byref(_pool(kr_pool)), kr_pool.shape[0],
                                          _ptr(block_table), max_pages, _ptr(seq_lens), B,
                                          _ptr(workspace), workspace.numel(), _ptr(out),
                                          _ptr(lse), _stream(stream)), "mla_prefill_attention")
    return out, lse


def prefill(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv, scale=0.0,
            workspace=None, out=None, lse=None, stream=None):
    """Prefill step through the decompress branch (both kernels). Returns (out, lse)."""
    dims = dims_for(q_c, q_r, w_uk, w_uv, ckv_pool.shape[1], scale)
    B, max_pages = block_table.shape
    M, H = q_c.shape[1], dims.num_heads
    if workspace is None:
        workspace = alloc_prefill_workspace(dims, B, max_pages, q_c.device)
    if out is None:
        out = torch.empty(B, M, H, dims.d_v, dtype=torch.bfloat16, device=q_c.device)
    if lse is None:
        lse = torch.empty(B, M, H, dtype=torch.float32, device=q_c.device)
    _b.check(_b.lib.mla_prefill(ctypes.byref(dims), _ptr(q_c), _ptr(q_r),
                                ctypes.byref(_pool(ckv_pool)), ctypes.byref(_pool(kr_pool)),
                                ckv_pool.shape[0], _ptr(block_table), max_pages, _ptr(seq_lens), B,
                                _ptr(w_uk), _ptr(w_uv), _ptr(workspace), workspace.numel(),
                                _ptr(out), _ptr(lse), _stream(stream)), "mla_prefill")
    return out, lse


def route(n_q, heads):
    """Which branch a step with n_q query tokens per sequence takes: "decompress" at or
    above the prefill threshold, or when the absorbed kernels cannot hold the
    n_q * heads query rows (more than 128); "absorb" otherwise."""
    if n_q >= PREFILL_THRESHOLD or n_q * heads > 128:
        return "decompress"
    return "absorb"


def attend(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv, scale=0.0,
           stream=None):
    """One attention step over the paged latent cache, routed by query count.
    Returns (out [B, n_q, H, d_v], lse [B, n_q, H])."""
    if route(q_c.shape[1], w_uk.shape[0]) == "decompress":
        return prefill(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv,
                       scale=scale, stream=stream)
    out, _, lse = decode(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv,
                         scale=scale, stream=stream)
    return out, lse
