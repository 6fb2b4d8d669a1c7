"""fp64 CPU oracle for absorbed MLA decode over a paged latent cache.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code with
the CUDA path; the only thing both sides share is the seeded input generator.

What it computes (page title, section):
  * ``decode_decompress`` -- the definition: per head, decompress
    K_nope = c_KV W_UK and V = c_KV W_UV, add the RoPE score, softmax with scale
    1/sqrt(d_n + d_R), weight V ("MLA operator design" §4 path A; "MHA2MLA" §2.1).
  * ``absorb_q`` -- q_c W_UK per head ("MLA operator design" §4 path B).
  * ``attend_latent`` -- scores against [c_KV | k_R], softmax, weighted sum of
    c_KV, plus the natural-log log-sum-exp; optionally over a token window.
  * ``combine`` -- log-sum-exp merge of partial results over disjoint windows.
  * ``absorb_out`` -- o_lat W_UV per head ("MHA2MLA" §2.1, v = c_kv W_uv).
  * ``decode_absorbed`` -- absorb_q -> attend_latent -> absorb_out, all fp64.
  * ``decompress_kv`` -- K_nope = c_KV W_UK and V = c_KV W_UV per head, for
    every cached token (the decompress branch, "MLA operator design" §3, §4).
  * ``prefill_decompress`` -- M causal queries per sequence through the
    decompress branch: decompress once per (sequence, head), then softmax over
    the visible tokens, with the natural-log log-sum-exp ("MLA operator design"
    §3, §6 prefill threshold; "MHA2MLA" §2.1).
  * ``gather`` -- the page-table gather, on raw bf16 bits.
  * ``e4m3_value`` / ``e4m3_encode`` / ``quantize_fp8_rows`` / ``dequant_fp8_rows``
    -- the low-precision latent cache: OCP E4M3 codes with one fp32 scale per
    cached token ("MLA operator design" introduction and §5 name a quantised
    cache gather; the format is the standard E4M3 one).
  * cache-size closed forms ("MLA operator design" §1, "MHA2MLA" §4.2).

Parity status: every function above is pinned by ``tests/test_oracle_pins.py``
(closed forms, special cases, invariants, brute force); none is unpinned.
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_num_threads.restype = i32
        lib.oracle_gather.argtypes = [P, i64, i64, i32, i32, i32, P, i32, P, i32, i32, P]
        lib.oracle_decode_decompress.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, f64,
                                                 P, P, P, P, i32, P, i32, P, P, P, P, i64, P]
        lib.oracle_absorb_q.argtypes = [i32, i32, i32, i32, P, P, P]
        lib.oracle_attend_latent.argtypes = [i32, i32, i32, i32, i32, i32, f64, P, P, P, P, i32,
                                             P, i32, P, i32, i32, P, i64, P, P]
        lib.oracle_combine.argtypes = [i64, i32, i32, P, P, P, P]
        lib.oracle_absorb_out.argtypes = [i32, i32, i32, i32, P, P, P, P]
        lib.oracle_rope.argtypes = [i32, i32, i32, P, P, ctypes.c_double, P]
        lib.oracle_rope.restype = i32
        lib.oracle_decompress_kv.argtypes = [i32, i32, i32, i32, i32, i32, P, i32, P, i32, P, P,
                                             P, i32, P, P]
        lib.oracle_prefill_decompress.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, f64,
                                                  P, P, P, P, i32, P, i32, P, P, P, P, i64, P, P]
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_value.restype = f64
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_quantize_fp8_rows.argtypes = [i64, i32, P, P, P]
        lib.oracle_quantize_fp8_rows.restype = None
        lib.oracle_dequant_fp8_rows.argtypes = [i64, i32, P, P, P]
        lib.oracle_dequant_fp8_rows.restype = None
        for name in ("oracle_gather", "oracle_decode_decompress", "oracle_absorb_q",
                     "oracle_attend_latent", "oracle_combine", "oracle_absorb_out",
                     "oracle_decompress_kv", "oracle_prefill_decompress"):
            getattr(lib, name).restype = i32
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (set OMP_NUM_THREADS before first use)."""
    return _load().oracle_num_threads()


# ----------------------------------------------------------------------------
# marshalling helpers (no arithmetic of the method)
# ----------------------------------------------------------------------------

def _bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array of bit patterns."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # plain PyTorch CPU, used as a container only
    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _i32(x) -> np.ndarray:
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _f64(x) -> np.ndarray:
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_bits_to_f64(x) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    u = _bits(x).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def default_scale(d_n: int, d_r: int) -> float:
    """Softmax scale 1/sqrt(d_hc + d_R) ("MLA operator design" §4)."""
    return 1.0 / math.sqrt(d_n + d_r)


def _sel(sel):
    if sel is None:
        return None, 0
    s = np.ascontiguousarray(np.asarray(sel, dtype=np.int64))
    return s, len(s)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


# ----------------------------------------------------------------------------
# public oracle functions
# ----------------------------------------------------------------------------

def gather(pool, block_table, seq_lens, page_size, max_len=None):
    """Bit copy of tokens [0, L_b) of each sequence from a paged pool.

    pool: bf16 [num_pages, P, width]. Returns uint16 [B, max_len, width]
    (zeros beyond L_b).
    """
    pb = _bits(pool)
    num_pages, P, width = pb.shape
    assert P == page_size
    bt, sl = _i32(block_table), _i32(seq_lens)
    B, max_pages = bt.shape
    max_len = int(sl.max()) if max_len is None else max_len
    out = np.zeros((B, max_len, width), dtype=np.uint16)
    rc = _load().oracle_gather(_p(pb), P * width, width, width, num_pages, P, _p(bt), max_pages,
                               _p(sl), B, max_len, _p(out))
    _check(rc, "gather")
    return out


def decode_decompress(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv,
                      scale=None, sel=None):
    """The definition, fp64. Returns out [B, n_q, H, d_v].

    sel: optional iterable of flat (b*n_q + i)*H + h indices to compute; other
    entries are left at zero.
    """
    qc, qr = _bits(q_c), _bits(q_r)
    B, n_q, H, d_n = qc.shape
    d_r = qr.shape[-1]
    ckv, kr = _bits(ckv_pool), _bits(kr_pool)
    num_pages, P, d_c = ckv.shape
    wuk, wuv = _bits(w_uk), _bits(w_uv)
    d_v = wuv.shape[-1]
    bt, sl = _i32(block_table), _i32(seq_lens)
    scale = default_scale(d_n, d_r) if scale is None else scale
    s, n_sel = _sel(sel)
    out = np.zeros((B, n_q, H, d_v), dtype=np.float64)
    rc = _load().oracle_decode_decompress(B, n_q, H, d_n, d_c, d_r, d_v, P, scale, _p(qc), _p(qr),
                                          _p(ckv), _p(kr), num_pages, _p(bt), bt.shape[1], _p(sl),
                                          _p(wuk), _p(wuv), _p(s), n_sel, _p(out))
    _check(rc, "decode_decompress")
    return out


def decompress_kv(ckv_pool, block_table, seq_lens, w_uk, w_uv, max_len=None):
    """K_nope [B, H, max_len, d_n] and V [B, H, max_len, d_v] in fp64 (rows past
    each sequence's length are zero)."""
    ckv = _bits(ckv_pool)
    num_pages, P, d_c = ckv.shape
    wuk, wuv = _bits(w_uk), _bits(w_uv)
    H, d_n, _ = wuk.shape
    d_v = wuv.shape[-1]
    bt, sl = _i32(block_table), _i32(seq_lens)
    B = sl.shape[0]
    max_len = int(sl.max()) if max_len is None else int(max_len)
    kn = np.zeros((B, H, max_len, d_n), dtype=np.float64)
    v = np.zeros((B, H, max_len, d_v), dtype=np.float64)
    rc = _load().oracle_decompress_kv(B, H, d_n, d_c, d_v, P, _p(ckv), num_pages, _p(bt),
                                      bt.shape[1], _p(sl), _p(wuk), _p(wuv), max_len, _p(kn), _p(v))
    _check(rc, "decompress_kv")
    return kn, v


def prefill_decompress(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv,
                       scale=None, sel=None):
    """Causal prefill through the decompress branch, fp64.

    q_c [B, M, H, d_n], q_r [B, M, H, d_r]: the last M tokens of each sequence.
    Returns (out [B, M, H, d_v], lse [B, M, H]); with sel, entries not selected
    are out = 0, lse = nan.
    """
    qc, qr = _bits(q_c), _bits(q_r)
    B, M, H, d_n = qc.shape
    d_r = qr.shape[-1]
    ckv, kr = _bits(ckv_pool), _bits(kr_pool)
    num_pages, P, d_c = ckv.shape
    wuk, wuv = _bits(w_uk), _bits(w_uv)
    d_v = wuv.shape[-1]
    bt, sl = _i32(block_table), _i32(seq_lens)
    scale = default_scale(d_n, d_r) if scale is None else scale
    s, n_sel = _sel(sel)
    out = np.zeros((B, M, H, d_v), dtype=np.float64)
    lse = np.full((B, M, H), np.nan, dtype=np.float64)
    rc = _load().oracle_prefill_decompress(B, M, H, d_n, d_c, d_r, d_v, P, scale, _p(qc),
                                           _p(qr), _p(ckv), _p(kr), num_pages, _p(bt),
                                           bt.shape[1], _p(sl), _p(wuk), _p(wuv), _p(s), n_sel,
                                           _p(out), _p(lse))
    _check(rc, "prefill_decompress")
    return out, lse


def absorb_q(q_c, w_uk):
    """q_lat = q_c W_UK per head, fp64. q_c [..., H, d_n] -> [..., H, d_c]."""
    qc = _bits(q_c)
    lead, (H, d_n) = qc.shape[:-2], qc.shape[-2:]
    wuk = _bits(w_uk)
    d_c = wuk.shape[-1]
    T = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (H, d_c), dtype=np.float64)
    _check(_load().oracle_absorb_q(T, H, d_n, d_c, _p(qc), _p(wuk), _p(out)), "absorb_q")
    return out


def rope(q_r, positions, theta=10000.0):
    """Rotary embedding of the RoPE part, fp64: consecutive pairs (2i, 2i+1)
    turn by positions[t] * theta^(-2i/d_r). q_r [..., H, d_r] bf16, positions
    [...] int (one per token) -> [..., H, d_r]."""
    x = _bits(q_r)
    lead, (H, d_r) = x.shape[:-2], x.shape[-2:]
    T = int(np.prod(lead)) if lead else 1
    pos = _i32(np.asarray(positions).reshape(-1))
    assert pos.size == T
    out = np.zeros(lead + (H, d_r), dtype=np.float64)
    _check(_load().oracle_rope(T, H, d_r, _p(x), _p(pos), float(theta), _p(out)), "rope")
    return out


def attend_latent(q, ckv_pool, kr_pool, block_table, seq_lens, scale, t_lo=0, t_hi=-1, sel=None):
    """Latent-space attention. q [B, n_q, H, d_c + d_r] as bf16 (tensor / uint16
    array) or float64 array. Returns (o_lat [B,n_q,H,d_c], lse [B,n_q,H])."""
    if isinstance(q, np.ndarray) and q.dtype == np.float64:
        qb, qf = None, np.ascontiguousarray(q)
        shape = qf.shape
    else:
        qb, qf = _bits(q), None
        shape = qb.shape
    B, n_q, H, D = shape
    ckv, kr = _bits(ckv_pool), _bits(kr_pool)
    num_pages, P, d_c = ckv.shape
    d_r = kr.shape[-1]
    assert D == d_c + d_r
    bt, sl = _i32(block_table), _i32(seq_lens)
    s, n_sel = _sel(sel)
    o = np.zeros((B, n_q, H, d_c), dtype=np.float64)
    lse = np.full((B, n_q, H), -np.inf, dtype=np.float64)
    rc = _load().oracle_attend_latent(B, n_q, H, d_c, d_r, P, scale, _p(qb), _p(qf), _p(ckv),
                                      _p(kr), num_pages, _p(bt), bt.shape[1], _p(sl), t_lo, t_hi,
                                      _p(s), n_sel, _p(o), _p(lse))
    _check(rc, "attend_latent")
    return o, lse


def combine(o_part, lse_part):
    """LSE merge. o_part [R, S, d_c], lse_part [R, S] (float64) -> (o [R,d_c], lse [R])."""
    op, lp = _f64(o_part), _f64(lse_part)
    R, S, d_c = op.shape
    o = np.zeros((R, d_c), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    _check(_load().oracle_combine(R, S, d_c, _p(op), _p(lp), _p(o), _p(lse)), "combine")
    return o, lse


def absorb_out(o_lat, w_uv):
    """out = o_lat W_UV per head. o_lat [..., H, d_c] as bf16 or float64."""
    if isinstance(o_lat, np.ndarray) and o_lat.dtype == np.float64:
        ob, of = None, np.ascontiguousarray(o_lat)
        shape = of.shape
    else:
        ob, of = _bits(o_lat), None
        shape = ob.shape
    lead, (H, d_c) = shape[:-2], shape[-2:]
    wuv = _bits(w_uv)
    d_v = wuv.shape[-1]
    T = int(np.prod(lead)) if lead else 1
    out = np.zeros(lead + (H, d_v), dtype=np.float64)
    _check(_load().oracle_absorb_out(T, H, d_c, d_v, _p(ob), _p(of), _p(wuv), _p(out)),
           "absorb_out")
    return out


def decode_absorbed(q_c, q_r, ckv_pool, kr_pool, block_table, seq_lens, w_uk, w_uv,
                    scale=None, sel=None):
    """Absorbed path in fp64 (no rounding between steps).

    Returns (out [B,n_q,H,d_v], o_lat [B,n_q,H,d_c], lse [B,n_q,H]).
    """
    qc = _bits(q_c)
    d_n = qc.shape[-1]
    qr64 = bf16_bits_to_f64(q_r)
    d_r = qr64.shape[-1]
    scale = default_scale(d_n, d_r) if scale is None else scale
    q_lat = absorb_q(qc, w_uk)
    q = np.ascontiguousarray(np.concatenate([q_lat, qr64], axis=-1))
    o_lat, lse = attend_latent(q, ckv_pool, kr_pool, block_table, seq_lens, scale, sel=sel)
    out = absorb_out(o_lat, w_uv)
    return out, o_lat, lse


# ----------------------------------------------------------------------------
# low-precision latent cache (E4M3 codes, one fp32 scale per row)
# ----------------------------------------------------------------------------

def e4m3_value(code) -> float:
    return _load().oracle_e4m3_value(int(code))


def e4m3_encode(y) -> int:
    return int(_load().oracle_e4m3_encode(float(np.float32(y))))


def quantize_fp8_rows(x):
    """x [..., d] bf16 -> (codes uint8 [..., d], scales float32 [...])."""
    xb = _bits(x)
    lead, d = xb.shape[:-1], xb.shape[-1]
    R = int(np.prod(lead)) if lead else 1
    codes = np.zeros(xb.shape, dtype=np.uint8)
    scales = np.zeros(lead, dtype=np.float32)
    _load().oracle_quantize_fp8_rows(R, d, _p(xb), _p(codes), _p(scales))
    return codes, scales


def dequant_fp8_rows(codes, scales):
    """(codes uint8 [..., d], scales float32 [...]) -> bf16 bit patterns (uint16) [..., d]."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    sc = np.ascontiguousarray(np.asarray(scales, dtype=np.float32))
    lead, d = c.shape[:-1], c.shape[-1]
    R = int(np.prod(lead)) if lead else 1
    out = np.zeros(c.shape, dtype=np.uint16)
    _load().oracle_dequant_fp8_rows(R, d, _p(c), _p(sc), _p(out))
    return out


def bf16_from_bits(bits):
    """uint16 bf16 bit patterns -> torch bfloat16 tensor (same shape)."""
    import torch
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)


# ----------------------------------------------------------------------------
# cache-size closed forms
# ----------------------------------------------------------------------------

def mla_cache_bytes_per_token(d_c: int, d_r: int, elem_bytes: int = 2) -> int:
    """Latent cache per token per layer: l * (d_R + d_c) elements ("MHA2MLA" §2.1)."""
    return (d_c + d_r) * elem_bytes


def mha_cache_bytes_per_token(n_heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """MHA cache per token per layer, K and V both stored: 2 * n_h * d_h elements."""
    return 2 * n_heads * head_dim * elem_bytes


def mha_key_bytes_per_token(n_heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """Bytes of one full-width per-head tensor per token (the 128x128 figure)."""
    return n_heads * head_dim * elem_bytes
