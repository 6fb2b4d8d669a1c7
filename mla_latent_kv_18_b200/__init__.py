"""B200 (sm_100a) MLA decode over a paged latent KV cache, by matrix absorption.

The public functions live in ``mla_latent_kv_18_b200.api`` and load the CUDA
library on first use (ImportError if it has not been built -- there is no CPU
fallback). ``mla_latent_kv_18_b200.inputs`` (seeded synthetic workloads) does
not need the library.
"""

_API = ("absorb_q", "decode_splitkv", "combine", "absorb_out", "decode", "Decoder", "dims_for",
        "make_dims", "get_device_error", "num_parts_for", "workspace_bytes", "plan")


def __getattr__(name):
    if name in _API:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
