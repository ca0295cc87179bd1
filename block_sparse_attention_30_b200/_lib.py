"""ctypes binding of the C ABI in include/vsa.h (libvsa.so, built in-tree).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libvsa.so.  Loading fails loudly when the library is missing;
there is no fallback implementation.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvsa.so")

VSA_OK = 0
STATUS_NAMES = {
    0: "VSA_OK", 1: "VSA_ERR_INVALID_ARGUMENT", 2: "VSA_ERR_UNSUPPORTED", 3: "VSA_ERR_WORKSPACE",
    4: "VSA_ERR_CUDA", 5: "VSA_ERR_TIMEOUT", 6: "VSA_ERR_DEVICE_CHECK",
}

# (name, restype, argtypes) for every entry point of include/vsa.h
_i, _sz, _p = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
_SHAPE = [_i] * 9                       # B, heads, head_dim, T, H, W, tt, th, tw
SIGNATURES = {
    "vsa_status_string": (ctypes.c_char_p, [_i]),
    "vsa_num_tiles": (_i, [_i] * 6),
    "vsa_workspace_bytes": (_sz, _SHAPE + [_i]),
    "vsa_workspace_init": (_i, [_p, _sz, _p]),
    "vsa_gather_tiles": (_i, [_p, _p] + _SHAPE + [_p]),
    "vsa_scatter_tiles": (_i, [_p, _p] + _SHAPE + [_p]),
    "vsa_select_blocks": (_i, [_p, _p] + _SHAPE + [_i, _p, _p, _sz, _p]),
    "vsa_linear_branch_fwd": (_i, [_p, _p, _p, _p] + [_i] * 6 + [_p, _sz, _p]),
    "vsa_sparse_attn_fwd": (_i, [_p] * 7 + _SHAPE + [_i, _p, _sz, _p]),
    "vsa_sparse_attn_fwd_train": (_i, [_p] * 7 + _SHAPE + [_i, _p, _sz, _p]),
    "vsa_sparse_attn_bwd": (_i, [_p] * 10 + _SHAPE + [_i, _p, _sz, _p]),
    "vsa_linear_branch_bwd": (_i, [_p] * 9 + [_i] * 7 + [_p, _sz, _p]),
    "vsa_quantize_qk_e4m3": (_i, [_p] * 6 + _SHAPE + [_p]),
    "vsa_sparse_attn_fwd_e4m3": (_i, [_p] * 7 + _SHAPE + [_i, _p, _sz, _p]),
    "vsa_sparse_linear_attn_fwd_e4m3": (_i, [_p] * 10 + _SHAPE + [_i, _p, _sz, _p]),
    "vsa_device_status": (_i, [_p, _p]),
    "vsa_select_blocks_noalloc": (_i, [_p, _p] + _SHAPE + [_i, _p, _p]),
    "vsa_selftest_wait_timeout": (_i, [_p, _sz, ctypes.c_uint, _p]),
}

# VSA_NOALLOC_SELECT_SCRATCH_BYTES of include/vsa.h
NOALLOC_SELECT_SCRATCH_BYTES = 32 * 1024 * 1024


class VSAError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


_lib = None


def lib():
    """Load libvsa.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m block_sparse_attention_30_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def check(fn, code):
    if code != VSA_OK:
        raise VSAError(fn, code)
