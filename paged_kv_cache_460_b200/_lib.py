"""ctypes loader for libpagedkv.so (C ABI declared in include/pagedkv.h).

There is no fallback: if the library is missing the import fails loudly, so no
code path can silently compute the decode step anywhere but in the CUDA kernels.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PKV_OK = 0
PKV_ERR_INVALID_ARG = 1
PKV_ERR_UNSUPPORTED = 2
PKV_ERR_CUDA = 3
PKV_ERR_NO_SPACE = 4
PKV_F16 = 0
PKV_BF16 = 1
PKV_I8 = 2
PKV_DEVERR_BAD_PAGE = 0x1
PKV_DEVERR_BAD_SLOT = 0x2
PKV_DEVERR_TIMEOUT = 0x4
PKV_MAX_DECODE_SPLITS = 4096

_lib = None

# name -> (restype, argtypes)
_P, _I, _I64, _D, _F, _SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double,
                             ctypes.c_float, ctypes.c_size_t)
SIGNATURES = {
    "pkv_status_string": (ctypes.c_char_p, [_I]),
    "kv_pool_create": (_I, [_I, _I, _I, _I, _I, _I, _P, _P, ctypes.POINTER(_P)]),
    "kv_pool_create_i8": (_I, [_I, _I, _I, _I, _I, _I, _P, _P, _P, _P, ctypes.POINTER(_P)]),
    "kv_pool_storage": (_I, [_P, ctypes.POINTER(_I)]),
    "kv_pool_destroy": (None, [_P]),
    "kv_pool_alloc": (_I, [_P, _I, _P]),
    "kv_pool_free": (_I, [_P, _I, _P]),
    "kv_pool_free_count": (_I, [_P]),
    "kv_pool_info": (_I, [_P, _P, _P, _P, _P, _P, _P]),
    "pkv_kv_cache_bytes": (_I64, [_I, _I, _I, _I64, _I]),
    "pkv_slot_mapping": (_I, [_P, _I, _P, _I, _I, _P]),
    "rope_apply": (_I, [_P, _P, _P, _I, _I, _I, _I, _D, _I, _P]),
    "paged_kv_append": (_I, [_P, _I, _P, _P, _P, _I, _P]),
    "rope_append": (_I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _D, _P]),
    "rope_append_step": (_I, [_P, _I, _P, _P, _P, _P, _I, _P, _I, _I, _D, _P]),
    "rms_norm": (_I, [_P, _P, _P, _P, _I, _I, _F, _I, _P]),
    "paged_prefill_attention": (_I, [_P, _I, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _F, _P]),
    "pkv_decode_default_splits": (_I, [_I, _I, _I, _I, _I, ctypes.POINTER(_I)]),
    "pkv_decode_auto_splits": (_I, [_P, _I, _I, _I, _I, ctypes.POINTER(_I)]),
    "pkv_decode_cluster_size": (_I, [_P, _I, _I, _I, _I, ctypes.POINTER(_I)]),
    "pkv_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "pkv_decode_workspace_clear": (_I, [_P, _SZ, _P]),
    "rope_table": (_I, [_P, _I, _I, _D, _P, _P]),
    "paged_decode_layer": (_I, [_P, _I, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _F, _I, _P, _SZ, _P]),
    "paged_decode_attention": (_I, [_P, _I, _P, _P, _P, _I, _P, _I, _I, _I, _F, _I, _P, _SZ, _P]),
    "paged_decode_attention_noalloc": (_I, [_P, _I, _P, _P, _P, _I, _P, _I, _I, _I, _F, _I, _P]),
    "kv_get_device_error": (_I, [ctypes.POINTER(ctypes.c_uint32)]),
}


class PagedKVError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (fn, status_string(status), status))


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libpagedkv.so is not built (%s); run `python -m paged_kv_cache_460_b200.build`"
                              % LIB_PATH)
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def status_string(status):
    return lib().pkv_status_string(int(status)).decode()


def check(fn, status):
    if status != PKV_OK:
        raise PagedKVError(fn, status)
