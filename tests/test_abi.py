"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and its host-side logic (partition plan, workspace sizing,
argument validation) behaves as documented. No kernel is launched here."""
import ctypes
import os
import random
import re

import pytest
import torch

from mla_latent_kv_18_b200 import build as mla_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def b():
    mla_build.build()
    from mla_latent_kv_18_b200 import _binding
    return _binding


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(b):
    declared = _declared()
    assert {"mla_absorb_q", "mla_decode_splitkv", "mla_combine", "mla_absorb_out"} <= declared
    for name in declared:
        assert hasattr(b.lib, name), name
    assert set(b.EXPORTS) == declared


def test_status_strings(b):
    for code, name in b.STATUS_NAMES.items():
        assert b.lib.mla_status_string(code).decode() == name
    assert b.lib.mla_status_string(99).decode() == "MLA_ERR_UNKNOWN"


def _dims(b, **kw):
    d = dict(num_heads=128, n_q=1, d_nope=128, d_latent=512, d_rope=64, d_v=128, page_size=64,
             softmax_scale=0.0)
    d.update(kw)
    return b.MLADims(**d)


# Virtual tiles the plan charges for each switch to another sequence inside a
# partition (a Q load and a partial-result write): 8 for 64-token tiles, 3 for
# 128-token tiles.
SWITCH_COST = {64: 8, 128: 3}


def _brute_plan(lens, max_pages, n_q, T, P):
    """The partition plan by enumeration: lay the tiles of the non-empty sequences
    end to end with SWITCH_COST[T] virtual positions between consecutive ones,
    cut the positions into P nearly equal ranges, and count for each sequence
    the ranges its real tiles fall in."""
    n = []
    for L in lens:
        L = max(0, min(L, max_pages * 64))
        n.append((L + T - 1) // T)
    N = sum(n)
    P = min(P, N) if N else P
    pos, seq_of_pos = 0, []           # cost position -> sequence (None for a virtual one)
    for b, nb in enumerate(n):
        if nb == 0:
            continue
        if seq_of_pos:
            seq_of_pos += [None] * SWITCH_COST[T]
        seq_of_pos += [b] * nb
    C = len(seq_of_pos)
    parts_of = [set() for _ in n]
    for p in range(P):
        for c in range(p * C // P, (p + 1) * C // P):
            if seq_of_pos[c] is not None:
                parts_of[seq_of_pos[c]].add(p)
    base = 0
    first, count, bases = [], [], []
    for b in range(len(n)):
        parts = sorted(parts_of[b])
        first.append(parts[0] if parts else -1)
        count.append(len(parts))
        bases.append(base)
        base += len(parts)
    return first, count, bases, base


@pytest.mark.parametrize("latent", [512, 64])
def test_plan_matches_brute_force(b, latent):
    from mla_latent_kv_18_b200 import api
    rng = random.Random(0)
    dims = _dims(b, d_latent=latent, d_rope=64 if latent == 512 else 8,
                 num_heads=128 if latent == 512 else 32, n_q=1 if latent == 512 else 2)
    T = 64 if latent == 512 else 128
    for trial in range(200):
        B = rng.randint(1, 40)
        max_pages = rng.randint(1, 40)
        lens = [rng.randint(dims.n_q, max_pages * 64) for _ in range(B)]
        P = rng.randint(1, 80)
        pf, cnt, base, total = api.plan(dims, lens, max_pages, P)
        e_first, e_cnt, e_base, e_total = _brute_plan(lens, max_pages, dims.n_q, T, P)
        assert pf.tolist() == e_first and cnt.tolist() == e_cnt and base.tolist() == e_base
        assert total == e_total <= B + P - 1


def test_num_parts_and_workspace(b):
    d = _dims(b)
    lib = b.lib
    assert lib.mla_decode_num_parts(ctypes.byref(d), 4, 148) == 1       # at least 8 tiles each
    assert lib.mla_decode_num_parts(ctypes.byref(d), 100, 148) == 13
    small = _dims(b, n_q=2, num_heads=32, d_nope=120, d_latent=64, d_rope=8)
    assert lib.mla_decode_num_parts(ctypes.byref(small), 100, 148) == 100   # one per SM at most
    assert lib.mla_decode_num_parts(ctypes.byref(small), 1000, 148) == 148
    assert lib.mla_decode_num_parts(ctypes.byref(d), 16 * 1024, 148) == 74
    assert lib.mla_decode_num_parts(ctypes.byref(d), 0, 148) == 1
    ws = lib.mla_decode_workspace_bytes(ctypes.byref(d), 16, 74)
    slots, R = 16 + 74, 128
    o = (slots * R * 512 * 4 + 255) // 256 * 256
    assert ws == o + (slots * R * 4 + 255) // 256 * 256
    bad = _dims(b, d_latent=256)
    assert lib.mla_decode_workspace_bytes(ctypes.byref(bad), 16, 74) == 0
    # the split-KV-named helpers are the same arithmetic
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 16, 74) == ws
    assert lib.mla_default_num_splits(ctypes.byref(d), 16, 65536, 148) == 74
    assert lib.mla_default_num_splits(ctypes.byref(d), 1, 256, 148) == 1
    for batch, L in ((3, 1000), (64, 32768), (2, 1)):
        tiles = batch * ((L + 63) // 64)
        assert lib.mla_default_num_splits(ctypes.byref(d), batch, L, 148) == \
            lib.mla_decode_num_parts(ctypes.byref(d), tiles, 148)
    r = _dims(b, n_q=2, num_heads=32, d_nope=120, d_latent=64, d_rope=8)
    assert lib.mla_default_num_splits(ctypes.byref(r), 32, 8192, 148) > 1
    assert lib.mla_default_num_splits(ctypes.byref(r), 32, 8192, 148) == \
        lib.mla_decode_num_parts(ctypes.byref(r), 32 * 64, 148)
    assert lib.mla_default_num_splits(ctypes.byref(bad), 16, 4096, 148) == 1


def test_argument_validation_without_launch(b):
    lib = b.lib
    d = _dims(b)
    null = ctypes.c_void_p(0)
    pool = b.MLAPool(0, 64 * 512, 512)
    # batch 0 is a no-op, checked before anything touches a device
    assert lib.mla_decode_splitkv(ctypes.byref(d), null, ctypes.byref(pool), ctypes.byref(pool),
                                  1, null, 1, null, 0, 1, null, 0, null) == 0
    # null pointers with work to do
    assert lib.mla_decode_splitkv(ctypes.byref(d), null, ctypes.byref(pool), ctypes.byref(pool),
                                  1, null, 1, null, 2, 1, null, 0, null) == 1
    # unsupported latent width
    d2 = _dims(b, d_latent=256)
    assert lib.mla_decode_splitkv(ctypes.byref(d2), null, ctypes.byref(pool), ctypes.byref(pool),
                                  1, null, 1, null, 2, 1, null, 0, null) == 2
    # too many query rows per sequence
    d3 = _dims(b, n_q=2)
    assert lib.mla_combine(ctypes.byref(d3), null, 0, null, 1, 2, 1, null, null, null) == 2
    # misaligned pointers are rejected before any launch
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1002)
    assert lib.mla_absorb_q(ctypes.byref(d), odd, fake, fake, fake, 4, null) == 1
    assert lib.mla_absorb_out(ctypes.byref(d), fake, odd, fake, 4, null) == 1
    assert lib.mla_absorb_q(ctypes.byref(d), fake, fake, fake, fake, -1, null) == 1
    assert lib.mla_absorb_q(ctypes.byref(d), null, null, null, null, 0, null) == 0
    ws_bytes = lib.mla_decode_workspace_bytes(ctypes.byref(d), 2, 1)
    bad_pool = b.MLAPool(0x1000, 64 * 512, 500)          # token stride below the width
    assert lib.mla_decode_splitkv(ctypes.byref(d), fake, ctypes.byref(bad_pool),
                                  ctypes.byref(bad_pool), 1, fake, 1, fake, 2, 1,
                                  ctypes.c_void_p(0x10000), ws_bytes, null) == 1
    good = b.MLAPool(0x1000, 64 * 576, 576)
    assert lib.mla_decode_splitkv(ctypes.byref(d), fake, ctypes.byref(good), ctypes.byref(good),
                                  1, fake, 1, fake, 2, 1, ctypes.c_void_p(0x10000), ws_bytes - 4,
                                  null) == 1                # workspace too small
    assert lib.mla_decode_splitkv(ctypes.byref(d), fake, ctypes.byref(good), ctypes.byref(good),
                                  1, fake, 1, fake, 2, 1, ctypes.c_void_p(0x10010), ws_bytes,
                                  null) == 1                # workspace not 256-byte aligned
    # the fused combine holds at most num_parts + 1 <= 160 slots per sequence in its
    # weight rows: 160 partitions are refused, 159 pass that check (and stop here at
    # the null workspace, before any device call)
    assert lib.mla_combine_absorb_out(ctypes.byref(d), null, 0, fake, 1, 2, 160, fake, fake, null,
                                      null) == 2
    assert lib.mla_combine_absorb_out(ctypes.byref(d), null, 0, fake, 1, 2, 159, fake, fake, null,
                                      null) == 1
    assert lib.mla_debug_wait_timeout(0, null) == 1


def test_prefill_workspace_size_and_validation_without_launch(b):
    lib = b.lib
    by = ctypes.byref
    d = _dims(b, n_q=300)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x1000)
    # K_nope then V, each [B, H, Lpad, 128] bf16 with Lpad = max_pages * 64 rounded up to 128
    for B, mp in ((2, 5), (8, 64), (1, 1), (3, 2)):
        l_pad = (mp * 64 + 127) // 128 * 128
        half = (B * 128 * l_pad * 128 * 2 + 255) // 256 * 256
        assert lib.mla_prefill_workspace_bytes(by(d), B, mp) == 2 * half
    # only the DeepSeek specialisation is compiled for the decompress branch
    dr = _dims(b, d_latent=64, d_rope=8, d_nope=120)
    assert lib.mla_prefill_workspace_bytes(by(dr), 2, 5) == 0
    pool = b.MLAPool(0x1000, 64 * 576, 576)
    kpool = b.MLAPool(0x1000, 64 * 64, 64)
    args = [fake, fake, by(pool), by(kpool), 4, fake, 2, fake, 2, fake, fake, fake, 1 << 30,
            fake, null, null]
    assert lib.mla_prefill(by(dr), *args) == 2
    assert lib.mla_prefill(by(_dims(b, n_q=300, page_size=16)), *args) == 2
    # batch 0 is a no-op; null pointers with work to do are rejected
    a0 = list(args)
    a0[8] = 0
    assert lib.mla_prefill(by(d), *a0) == 0
    a1 = list(args)
    a1[0] = null
    assert lib.mla_prefill(by(d), *a1) == 1
    ws = lib.mla_prefill_workspace_bytes(by(d), 2, 2)
    assert lib.mla_decompress_kv(by(d), by(pool), 4, fake, 2, fake, 2, fake, fake, fake, ws - 2,
                                 null) == 1                 # workspace too small
    assert lib.mla_decompress_kv(by(d), by(pool), 4, fake, 2, fake, 2, fake, fake,
                                 ctypes.c_void_p(0x1010), ws, null) == 1   # not 256-B aligned
    assert lib.mla_prefill_attention(by(d), ctypes.c_void_p(0x1002), fake, by(kpool), 4, fake, 2,
                                     fake, 2, fake, ws, fake, null, null) == 1   # misaligned q_c
    # mla_prefill checks the attention step's arguments before launching the decompression:
    # everything valid except a misaligned output is refused without touching a device
    wsp = ctypes.c_void_p(0x100000)
    ok_args = [fake, fake, by(pool), by(kpool), 4, fake, 2, fake, 2, fake, fake, wsp, ws]
    assert lib.mla_prefill(by(d), *ok_args, ctypes.c_void_p(0x1008), null, null) == 1
    assert lib.mla_prefill(by(d), *ok_args, fake, ctypes.c_void_p(0x1002), null) == 1


def test_cache_write_and_fp8_calls_validate_without_launch(b):
    lib = b.lib
    by = ctypes.byref
    d = _dims(b)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x1000)
    cpool = b.MLAPool(0x1000, 64 * 512, 512)
    kpool = b.MLAPool(0x1000, 64 * 64, 64)
    c8 = b.MLAPool(0x1000, 64 * 512, 512)
    # no tokens: nothing to do; null pointers with tokens: rejected
    assert lib.mla_append_kv(by(d), null, null, null, null, 0, 10000.0, by(cpool), by(kpool), 4,
                             null, 2, 2, null) == 0
    assert lib.mla_append_kv(by(d), null, fake, fake, fake, 3, 10000.0, by(cpool), by(kpool), 4,
                             fake, 2, 2, null) == 1
    assert lib.mla_append_kv(by(d), fake, fake, fake, fake, 3, float("nan"), by(cpool), by(kpool),
                             4, fake, 2, 2, null) == 1      # theta must be finite
    assert lib.mla_append_kv(by(_dims(b, page_size=32)), fake, fake, fake, fake, 3, 10000.0,
                             by(cpool), by(kpool), 4, fake, 2, 2, null) == 2   # page size other than 64
    # the E4M3 cache: latent width a multiple of 16, scales given, 16-byte strides
    assert lib.mla_append_kv_fp8(by(_dims(b, d_latent=72)), fake, fake, fake, fake, 3, 1e4,
                                 by(c8), fake, by(kpool), 4, fake, 2, 2, null) == 2
    assert lib.mla_append_kv_fp8(by(d), fake, fake, fake, fake, 3, 1e4, by(c8), null, by(kpool),
                                 4, fake, 2, 2, null) == 1
    odd = b.MLAPool(0x1000, 64 * 520, 520)
    assert lib.mla_append_kv_fp8(by(d), fake, fake, fake, fake, 3, 1e4, by(odd), fake, by(kpool),
                                 4, fake, 2, 2, null) == 1
    # dequantising gather: width, alignment, no-op sizes
    assert lib.mla_gather_dequant_fp8(by(c8), fake, 24, 4, fake, 2, fake, 2, 10, fake, null) == 2
    assert lib.mla_gather_dequant_fp8(by(c8), fake, 512, 4, fake, 2, fake, 2, 10,
                                      ctypes.c_void_p(0x1008), null) == 1
    assert lib.mla_gather_dequant_fp8(by(c8), fake, 512, 4, fake, 2, fake, 0, 10, fake, null) == 0
    assert lib.mla_gather_dequant_fp8(by(c8), fake, 512, 4, fake, 2, fake, 2, 0, fake, null) == 0
    # decompress from the E4M3 cache: scales required, token stride at least the width
    dp = _dims(b, n_q=300)
    ws = lib.mla_prefill_workspace_bytes(by(dp), 2, 2)
    assert lib.mla_decompress_kv_fp8(by(dp), by(c8), null, 4, fake, 2, fake, 2, fake, fake, fake,
                                     ws, null) == 1
    short = b.MLAPool(0x1000, 64 * 256, 256)
    assert lib.mla_decompress_kv_fp8(by(dp), by(short), fake, 4, fake, 2, fake, 2, fake, fake,
                                     fake, ws, null) == 1



def test_fp8_decode_validates_without_launch(b):
    lib = b.lib
    by = ctypes.byref
    d = _dims(b)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x1000)
    kpool = b.MLAPool(0x1000, 64 * 64, 64)
    c8 = b.MLAPool(0x1000, 64 * 512, 512)
    P = 4
    ws = lib.mla_decode_workspace_bytes(by(d), 2, P)

    def call(dims=d, q=fake, codes=c8, scales=fake, kr=kpool, batch=2, parts=P, wsb=ws,
             workspace=fake):
        return lib.mla_decode_splitkv_fp8(by(dims), q, by(codes), scales, by(kr), 8, fake, 4, fake,
                                          batch, parts, workspace, wsb, null)

    # the 64-wide latent variant has no E4M3 decode
    small = _dims(b, num_heads=32, n_q=2, d_nope=120, d_latent=64, d_rope=8)
    assert call(dims=small, wsb=lib.mla_decode_workspace_bytes(by(small), 2, P)) == 2
    assert call(batch=0) == 0                                           # no-op
    assert call(scales=null) == 1                                       # scales required
    assert call(scales=ctypes.c_void_p(0x1004)) == 1                    # 16-byte aligned (TMA)
    assert call(codes=b.MLAPool(0x1008, 64 * 512, 512)) == 1            # 16-byte base
    assert call(codes=b.MLAPool(0x1000, 64 * 520, 520)) == 1            # 16-byte strides
    assert call(codes=b.MLAPool(0x1000, 64 * 256, 256)) == 1            # token stride >= 512
    assert call(codes=b.MLAPool(0x1000, 32 * 512, 512)) == 1            # page holds 64 tokens
    assert call(wsb=ws - 1) == 1                                        # workspace too small
    assert call(workspace=ctypes.c_void_p(0x1010)) == 1                 # 256-byte aligned
    assert call(q=null) == 1

def test_noalloc_decode_checks_outputs_before_launching(b):
    # a misaligned or missing o_lat (or lse_out) is refused before the split-KV decode is
    # launched, so nothing touches a device
    lib = b.lib
    by = ctypes.byref
    d = _dims(b)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x1000)
    pool = b.MLAPool(0x1000, 64 * 576, 576)
    args = [fake, by(pool), by(pool), 4, fake, 2, fake, 2, 4]
    assert lib.mla_decode_latent_noalloc(by(d), *args, null, null, null) == 1
    assert lib.mla_decode_latent_noalloc(by(d), *args, ctypes.c_void_p(0x1004), null, null) == 1
    assert lib.mla_decode_latent_noalloc(by(d), *args, fake, ctypes.c_void_p(0x1002), null) == 1
