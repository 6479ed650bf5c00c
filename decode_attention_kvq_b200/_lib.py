"""ctypes loader for libkvq.so with the prototypes of include/kvq.h."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python decode_attention_kvq_b200/build.py` "
        "(the CUDA library is required; there is no CPU fallback)")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float

_PROTOS = {
    "kvq_append": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _P, _P]),
    "kvq_append_paged": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _I, _I,
                              _P, _P]),
    "kvq_append_calibrate": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _P, _P]),
    "kvq_append_mixed": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _P, _P, _I,
                              _P, _P]),
    "kvq_decode_attn_mixed": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _I, _P, _I, _F, _P, _P,
                                   _SZ, _I, _P, _P]),
    "kvq_mixed_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "kvq_decode_attn": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _I, _F, _P, _P, _SZ, _I, _P, _P]),
    "kvq_append_decode": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _F, _P, _P, _SZ, _I,
                               _P, _P]),
    "kvq_decode_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "kvq_chunk_attn": (_I, [_P, _I, _I, _I, _I, _I, _I, _P, _P, _I, _F, _P, _P, _SZ, _I, _P,
                            _P]),
    "kvq_chunk_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "kvq_window_attn": (_I, [_P, _I, _I, _I, _I, _I, _I, _P, _P, _I, _I, _F, _P, _P, _SZ, _I,
                             _P, _P]),
    "kvq_window_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "kvq_decode_plan": (_I, [_I, _I, _I, _I, _I, _P, _P]),
    "kvq_dequant": (_I, [_P, _P, _I64, _I, _I, _P, _P]),
    "kvq_status_string": (ctypes.c_char_p, [_I]),
    "kvq_read_error": (_I, [_P, _P, _P]),
    "kvq_check_error": (_I, [_P, _P]),
    "kvq_cache_bytes": (_I64, [_I64, _I64, _I64, _I, _I]),
    "kvq_version": (ctypes.c_char_p, []),
    "kvq_decode_attn_noalloc": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _I, _F, _P, _I, _P, _P]),
    "kvq_noalloc_scratch_bytes": (_SZ, []),
    "kvq_pager_bytes": (_SZ, [_I, _I, _I, _I]),
    "kvq_pager_init": (_I, [_P, _SZ, _I, _I, _I, _I, _P, _I, _P]),
    "kvq_pager_append": (_I, [_P, _I, _I64, _P]),
    "kvq_pager_popn": (_I64, [_P, _I, _I64]),
    "kvq_pager_release": (_I, [_P, _I]),
    "kvq_pager_reset": (None, [_P]),
    "kvq_pager_free_pages": (_I, [_P]),
    "kvq_pager_pages_used": (_I, [_P, _I]),
    "kvq_pager_seq_len": (_I64, [_P, _I]),
    "kvq_pager_table": (_P, [_P]),
    "kvq_pager_lens": (_P, [_P]),
}

for _name, (_res, _args) in _PROTOS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.kvq_status_string(status).decode()} ({status})")


def check(status: int, where: str) -> None:
    if status != 0:
        raise KvqError(status, where)
