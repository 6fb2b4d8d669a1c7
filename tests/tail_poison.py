"""Non-finite page tails for the cache tests.

A paged cache fills a sequence's last page only up to its length; the rest of
that page holds whatever was there (an unwritten slot of a pool allocated
without clearing, or a recycled page), possibly NaN or infinity bit patterns.
The kernels load whole pages, so they must keep those rows out of every result.
"""
import torch

_SPECIALS = (float("nan"), float("inf"), float("-inf"))


def poison_page_tails(inp, page_size=64):
    """Copy of an input dict whose pools hold NaN, +Inf and -Inf (cycling over
    rows and channels) in every row past a sequence's end in its last page."""
    ckv, kr = inp["ckv_pool"].clone(), inp["kr_pool"].clone()
    specials = torch.tensor(_SPECIALS, dtype=torch.float32)
    for b, L in enumerate(inp["seq_lens"].tolist()):
        used = L % page_size
        if L == 0 or used == 0:
            continue
        page = int(inp["block_table"][b, (L - 1) // page_size])
        rows = torch.arange(used, page_size)
        for pool in (ckv, kr):
            idx = (rows[:, None] + torch.arange(pool.shape[-1])[None, :]) % len(_SPECIALS)
            pool[page, used:] = specials[idx].to(pool.dtype)
    out = dict(inp)
    out["ckv_pool"], out["kr_pool"] = ckv, kr
    return out
