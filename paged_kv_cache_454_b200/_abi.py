"""ctypes view of ``libpa.so`` (declared in ``include/pa.h``).

Only argument marshalling lives here; every step of the computation runs in the
library's CUDA kernels.  Loading fails loudly when the library has not been
built: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpa.so")

PA_OK = 0
PA_ERR_ARG = 1
PA_ERR_SHAPE = 2
PA_ERR_UNSUPPORTED = 3
PA_ERR_WORKSPACE = 4
PA_ERR_CUDA = 5
PA_ERR_NO_BLOCKS = 6

PA_SWAP_OUT = 0
PA_SWAP_IN = 1

PA_DEV_ERR_BLOCK_ID = 0x1
PA_DEV_ERR_SLOT = 0x2
PA_DEV_ERR_CONTEXT = 0x4
PA_DEV_ERR_TIMEOUT = 0x8

PA_KERNEL_AUTO = 0
PA_KERNEL_SIMT = 1
PA_KERNEL_TCGEN05 = 2
PA_PREFILL_EXACT_WEIGHTS = 0x1

PA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

# Every entry point of include/pa.h, with its ctypes signature.
c_int, c_i32, c_i64, c_f32 = ctypes.c_int, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
c_vp, c_size = ctypes.c_void_p, ctypes.c_size_t


class PoolDesc(ctypes.Structure):
    _fields_ = [("num_blocks", c_i32), ("num_kv_heads", c_i32), ("block_size", c_i32),
                ("head_dim", c_i32)]


SIGNATURES = {
    "pa_reshape_and_cache": (c_int, [c_vp, c_vp, c_i64, c_vp, c_vp, PoolDesc, c_vp, c_i32, c_vp]),
    "pa_copy_blocks": (c_int, [c_vp, c_vp, PoolDesc, c_vp, c_i32, c_vp]),
    "pa_decode_workspace_size": (c_size, [c_i32, c_i32, PoolDesc, c_i32]),
    "pa_decode": (c_int, [c_vp, c_i64, c_vp, c_vp, PoolDesc, c_vp, c_i32, c_vp, c_i32, c_i32,
                          c_f32, c_vp, c_vp, c_vp, c_size, c_vp]),
    "pa_decode_workspace_size_ex": (c_size, [c_i32, c_i32, PoolDesc, c_i32, c_i32]),
    "pa_decode_ex": (c_int, [c_vp, c_i64, c_vp, c_vp, PoolDesc, c_vp, c_i32, c_vp, c_i32, c_i32,
                             c_f32, c_vp, c_vp, c_vp, c_size, c_i32, c_i32, c_vp]),
    "pa_decode_noalloc": (c_int, [c_vp, c_i64, c_vp, c_vp, PoolDesc, c_vp, c_i32, c_vp, c_i32,
                                  c_i32, c_f32, c_vp, c_vp, c_vp]),
    "pa_chunked_prefill": (c_int, [c_vp, c_i64, c_vp, c_i32, c_i32, c_vp, c_vp, PoolDesc, c_vp,
                                   c_i32, c_vp, c_i32, c_i32, c_f32, c_vp, c_vp, c_vp]),
    "pa_chunked_prefill_ex": (c_int, [c_vp, c_i64, c_vp, c_i32, c_i32, c_vp, c_vp, PoolDesc, c_vp,
                                      c_i32, c_vp, c_i32, c_i32, c_f32, c_vp, c_vp, ctypes.c_uint32,
                                      c_vp]),
    "pa_gather_kv": (c_int, [c_vp, c_vp, PoolDesc, c_vp, c_i32, c_vp, c_vp, c_i32, c_i32, c_vp,
                             c_vp, c_vp]),
    "pa_get_device_error": (c_int, [ctypes.POINTER(ctypes.c_uint32), c_vp]),
    "pa_status_string": (ctypes.c_char_p, [c_int]),
    "pa_abi_version": (c_int, []),
    # fused sampler (include/pa_sampler.h)
    "pa_sample": (c_int, [c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    # host KV-cache block manager (include/pa_kv_manager.h)
    "pa_kvm_create": (c_vp, [c_i32, c_i32, c_i32, c_i32]),
    "pa_kvm_destroy": (None, [c_vp]),
    "pa_kvm_num_free_blocks": (c_i32, [c_vp]),
    "pa_kvm_add_sequence": (c_int, [c_vp, c_i64, c_vp, c_i32, c_vp, c_vp]),
    "pa_kvm_append_tokens": (c_int, [c_vp, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp]),
    "pa_kvm_decode_step": (c_int, [c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "pa_kvm_fork": (c_int, [c_vp, c_i64, c_i64]),
    "pa_kvm_share_prefix": (c_int, [c_vp, c_i64, c_i64, c_i32]),
    "pa_kvm_share_blocks": (c_int, [c_vp, c_i64, c_i64, c_vp, c_i32]),
    "pa_kvm_free_sequence": (c_int, [c_vp, c_i64]),
    "pa_kvm_sequence_info": (c_int, [c_vp, c_i64, c_vp, c_vp]),
    "pa_kvm_block_table": (c_int, [c_vp, c_i64, c_vp, c_i32]),
    "pa_kvm_batch": (c_int, [c_vp, c_vp, c_i32, c_i32, c_vp, c_vp]),
    "pa_kvm_batch_update": (c_int, [c_vp, c_vp, c_i32, c_i32, c_vp, c_vp]),
    "pa_kvm_ref_count": (c_i32, [c_vp, c_i32]),
    "pa_kvm_swap_out": (c_int, [c_vp, c_i64, c_vp, c_i32, c_vp]),
    "pa_kvm_swap_in": (c_int, [c_vp, c_i64, c_vp, c_i32, c_vp]),
    "pa_kvm_num_free_host_blocks": (c_i32, [c_vp]),
    # block swapping (include/pa_swap.h)
    "pa_swap_blocks": (c_int, [c_vp, c_vp, PoolDesc, c_vp, c_vp, c_i32, c_vp, c_i32, c_i32, c_vp]),
    # paged read-bandwidth probe (include/pa_probe.h)
    "pa_read_probe": (c_int, [c_vp, c_vp, PoolDesc, c_vp, c_i32, c_vp, c_i32, c_vp, c_i32, c_vp]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpa.so and attach the signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m paged_kv_cache_454_b200.build` "
            "(there is no non-CUDA fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


class PaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = load().pa_status_string(status)
        super().__init__(f"{fn} failed: {msg.decode() if msg else status}")


def check(fn: str, status: int) -> None:
    if status != PA_OK:
        raise PaError(fn, status)
