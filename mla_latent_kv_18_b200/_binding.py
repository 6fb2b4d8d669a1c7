"""ctypes binding of ``libmla_b200.so`` (the C ABI in include/mla_decode.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
Importing this module loads the library and raises ``ImportError`` if it is
missing -- there is no fallback.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_b200.so")

MLA_OK = 0
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_CUDA",
                4: "MLA_ERR_DEVICE_BOUNDS", 5: "MLA_ERR_TIMEOUT"}

EXPORTS = ("mla_absorb_q", "mla_decode_num_parts", "mla_decode_workspace_bytes",
           "mla_decode_splitkv", "mla_combine", "mla_absorb_out", "mla_get_device_error",
           "mla_status_string", "mla_decode_plan", "mla_debug_wait_timeout",
           "mla_decode_latent_noalloc", "mla_debug_gather", "mla_combine_absorb_out",
           "mla_absorb_q_rope", "mla_prefill_workspace_bytes", "mla_decompress_kv",
           "mla_prefill_attention", "mla_prefill", "mla_append_kv",
           "mla_append_kv_fp8", "mla_gather_dequant_fp8", "mla_decompress_kv_fp8",
           "mla_default_num_splits", "mla_decode_workspace_size", "mla_decode_splitkv_fp8")


class MLADims(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("n_q", ctypes.c_int32), ("d_nope", ctypes.c_int32),
                ("d_latent", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


class MLAPool(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("page_stride", ctypes.c_int64),
                ("token_stride", ctypes.c_int64)]


class MLAError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library not built: {LIB_PATH} (run python -m "
                          "mla_latent_kv_18_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    D = ctypes.POINTER(MLADims)
    PL = ctypes.POINTER(MLAPool)
    sig = {
        "mla_absorb_q": (i32, [D, P, P, P, P, i32, P]),
        "mla_decode_num_parts": (i32, [D, i64, i32]),
        "mla_decode_workspace_bytes": (sz, [D, i32, i32]),
        "mla_decode_splitkv": (i32, [D, P, PL, PL, i32, P, i32, P, i32, i32, P, sz, P]),
        "mla_combine": (i32, [D, P, sz, P, i32, i32, i32, P, P, P]),
        "mla_absorb_out": (i32, [D, P, P, P, i32, P]),
        "mla_get_device_error": (i32, [ctypes.POINTER(i32), P]),
        "mla_status_string": (ctypes.c_char_p, [i32]),
        "mla_decode_plan": (i64, [D, P, i32, i32, i32, P, P, P]),
        "mla_debug_wait_timeout": (i32, [i64, P]),
        "mla_decode_latent_noalloc": (i32, [D, P, PL, PL, i32, P, i32, P, i32, i32, P, P, P]),
        "mla_debug_gather": (i32, [PL, i32, i32, P, i32, P, i32, i32, P, P]),
        "mla_combine_absorb_out": (i32, [D, P, sz, P, i32, i32, i32, P, P, P, P]),
        "mla_absorb_q_rope": (i32, [D, P, P, P, P, ctypes.c_float, P, i32, P]),
        "mla_prefill_workspace_bytes": (sz, [D, i32, i32]),
        "mla_decompress_kv": (i32, [D, PL, i32, P, i32, P, i32, P, P, P, sz, P]),
        "mla_prefill_attention": (i32, [D, P, P, PL, i32, P, i32, P, i32, P, sz, P, P, P]),
        "mla_prefill": (i32, [D, P, P, PL, PL, i32, P, i32, P, i32, P, P, P, sz, P, P, P]),
        "mla_append_kv": (i32, [D, P, P, P, P, i32, ctypes.c_float, PL, PL, i32, P, i32, i32, P]),
        "mla_append_kv_fp8": (i32, [D, P, P, P, P, i32, ctypes.c_float, PL, P, PL, i32, P, i32, i32,
                                    P]),
        "mla_gather_dequant_fp8": (i32, [PL, P, i32, i32, P, i32, P, i32, i32, P, P]),
        "mla_decompress_kv_fp8": (i32, [D, PL, P, i32, P, i32, P, i32, P, P, P, sz, P]),
        "mla_default_num_splits": (i32, [D, i32, i32, i32]),
        "mla_decode_workspace_size": (sz, [D, i32, i32]),
        "mla_decode_splitkv_fp8": (i32, [D, P, PL, P, PL, i32, P, i32, P, i32, i32, P, sz, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def check(status, what):
    if status != MLA_OK:
        raise MLAError(status, what)
