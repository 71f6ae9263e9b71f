"""ctypes loader for ``libulysses_b200.so`` (built in-tree by ``build.py``).

There is no fallback: if the library is missing or does not load, every
entry point raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libulysses_b200.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape or option", 3: "CUDA runtime error",
          4: "bounded device wait timed out"}

MAX_RANKS = 16


class UlyssesError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} (status {code})")
        self.code = code


_lib = None

_vpp = ctypes.POINTER(ctypes.c_void_p)
_fpp = ctypes.POINTER(ctypes.c_void_p)
_i64 = ctypes.c_int64
_i = ctypes.c_int
_v = ctypes.c_void_p

_SIGS = {
    "ulysses_a2a_seq_to_head": [_vpp, _vpp, _vpp, _vpp, _vpp, _vpp, _i64, _i, _i, _i, _i, _v, _i, _i, _i, _v],
    "ulysses_a2a_head_to_seq": [_vpp, _vpp, _vpp, _vpp, _vpp, _vpp, _i64, _i, _i, _i, _i, _v, _i, _i, _i, _v],
    "ulysses_a2a_seq_to_head_frag": [_vpp, _vpp, _vpp, _v, _v, _v, _i64, _i, _i, _i, _i, _i, _i, _v],
    "ulysses_a2a_head_to_seq_frag": [_v, _v, _v, _vpp, _vpp, _vpp, _i64, _i, _i, _i, _i, _i, _i, _v],
    "ulysses_a2a_pack": [_v, _v, _v, _v, _v, _v, _i64, _i, _i, _i, _i, _i, _i, _v],
    "ulysses_a2a_unpack": [_v, _v, _v, _v, _v, _v, _i64, _i, _i, _i, _i, _i, _i, _v],
    "ulysses_qkv_proj_seq_to_head": [_vpp, _v, _vpp, _vpp, _vpp, _i64, _i, _i, _i, _i, _i, _v],
    "ulysses_out_proj_head_to_seq": [_vpp, _v, _vpp, _i64, _i, _i, _i, _i, _i, _v],
    "ulysses_out_proj_bwd": [_vpp, _v, _vpp, _vpp, _v, _i64, _i, _i, _i, _i, _i, _v],
    "ulysses_qkv_proj_bwd": [_vpp, _v, _vpp, _vpp, _vpp, _vpp, _v, _i64, _i, _i, _i, _i, _i, _v],
    "ulysses_attn_fwd": [_vpp, _vpp, _vpp, _vpp, _fpp, _i64, _i, _i, _i, _i, _v, _i, _i, ctypes.c_float, _i,
                         _i, _i, _v],
    "ulysses_attn_bwd_workspace_size": [_i64, _i, _i, _i, _i, _i],
    "ulysses_attn_bwd_seq_workspace_size": [_i64, _i, _i, _i, _i, _i],
    "ulysses_attn_bwd": [_vpp, _vpp, _vpp, _vpp, _fpp, _vpp, _vpp, _vpp, _vpp, _i64, _i, _i, _i, _i, _v, _i, _i,
                         ctypes.c_float, _i, _v, ctypes.c_size_t, _i, _i, _v],
    "ulysses_status_string": [_i],
    "ulysses_get_device_status": [_v, ctypes.POINTER(ctypes.c_uint32)],
    "ulysses_set_wait_limit": [ctypes.c_uint32],
    "ulysses_selftest_bounded_wait": [_v],
    "ulysses_attn_bwd_onepass_layout_fits": [ctypes.c_uint32],
    "ulysses_attn_fwd_seq": [_vpp, _vpp, _vpp, _vpp, _fpp, _i64, _i, _i, _i, _i, _v, _i, _i, ctypes.c_float, _i,
                             _i, _i, _v],
    "ulysses_attn_bwd_seq": [_vpp, _vpp, _vpp, _vpp, _fpp, _vpp, _vpp, _vpp, _vpp, _i64, _i, _i, _i, _i, _v, _i,
                             _i, ctypes.c_float, _i, _v, ctypes.c_size_t, _i, _i, _v],
    "ulysses_attn_bwd_noalloc": [_vpp, _vpp, _vpp, _vpp, _fpp, _vpp, _vpp, _vpp, _vpp, _i64, _i, _i, _i, _i, _v, _i,
                                 _i, ctypes.c_float, _i, _i, _v],
    "ulysses_host_pipeline_scratch_bytes": [_i64, _i, _i, _i, _i, _i, _i],
    "ulysses_host_pipeline_create": [_i64, _i, _i, _i, _i, _i, _i, _v, ctypes.c_size_t, ctypes.POINTER(_v)],
    "ulysses_host_pipeline_submit": [_v, _vpp, _vpp, _vpp, _vpp, _vpp, _vpp, _vpp, _vpp, _v, _i, ctypes.c_float,
                                     _v, _v],
    "ulysses_host_pipeline_synchronize": [_v],
    "ulysses_host_pipeline_destroy": [_v],
}
_RES = {"ulysses_attn_bwd_workspace_size": ctypes.c_size_t, "ulysses_attn_bwd_seq_workspace_size": ctypes.c_size_t, "ulysses_status_string": ctypes.c_char_p,
        "ulysses_set_wait_limit": None, "ulysses_host_pipeline_scratch_bytes": ctypes.c_size_t}


def lib():
    """The loaded library (loads on first use; raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m ulysses_sequence_parallelism_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = _RES.get(name, ctypes.c_int)
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def check(fn, code):
    if code != 0:
        raise UlyssesError(fn, code)
