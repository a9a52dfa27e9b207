"""ctypes binding of libsa.so: one Python function per C entry point, same names.

Argument marshalling only: pointers are plain integers (device addresses, or
host addresses for the introspection calls), streams are cudaStream_t handles
as integers. Every compute step runs in the library's CUDA kernels; if the
library is missing this module raises instead of falling back to anything.
"""

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
# SA_LIBRARY=checked selects the checked build (device-side bounds checks,
# include/sa.h: sa_build_info); the default is the release build.
LIB_PATH = os.path.join(HERE, "libsa_checked.so" if os.environ.get("SA_LIBRARY") == "checked"
                        else "libsa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "sa.h")

SA_OK = 0
SA_ERR_INVALID_ARG = 1
SA_ERR_STATE = 2
SA_ERR_UNSUPPORTED = 3
SA_ERR_CUDA = 4
SA_ERR_TIMEOUT = 5
SA_ERR_RANGE = 6
SA_ERR_BOUNDS = 7
SA_BUILD_DEVICE_CHECKS = 1
SA_TIER_NOISY = 0
SA_TIER_CLEAN = 1
SA_MAX_ATTENDED = 16
SA_NOALLOC_MAX_KEY_BYTES = 64 << 20
SA_PAYLOAD_FP8 = 0
SA_PAYLOAD_BF16 = 1
SA_IPC_HANDLE_BYTES = 64


class SaConfig(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("frames_per_chunk", ctypes.c_int32),
        ("tok_h", ctypes.c_int32),
        ("tok_w", ctypes.c_int32),
        ("sink_chunks", ctypes.c_int32),
        ("window_chunks", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("rope_theta", ctypes.c_float),
        ("ref_frames", ctypes.c_int32),
    ]


class SaError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{status_name(status)}: {message}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_I32P = ctypes.POINTER(ctypes.c_int32)
_CFGP = ctypes.POINTER(SaConfig)

_SIGNATURES = {
    "sa_validate_config": (_I, [_CFGP]),
    "sa_required_bytes": (ctypes.c_size_t, [_CFGP]),
    "sa_create": (_I, [_CFGP, _P, ctypes.c_size_t, ctypes.POINTER(_P)]),
    "sa_destroy": (_I, [_P]),
    "sa_reset": (_I, [_P]),
    "sa_append_chunk": (_I, [_P, _I, _P, _P, _P]),
    "sa_append_chunk_frames": (_I, [_P, _I, _P, _P, _I, _P]),
    "sa_set_reference": (_I, [_P, _P, _P, _P]),
    "sa_attend": (_I, [_P, _P, _P, _P, _I, _P, _P, _P]),
    "sa_attend_frames": (_I, [_P, _P, _P, _P, _I, _I, _P, _P, _P]),
    "sa_attend_aligned": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P]),
    "sa_stage_keys": (_I, [_P, _P, _P]),
    "sa_stage_keys_frames": (_I, [_P, _P, _I, _P]),
    "sa_attend_staged": (_I, [_P, _P, _P, _I, _P, _P, _P]),
    "sa_debug_attend_simt": (_I, [_P, _P, _P, _P, _I, _P, _P, _P]),
    "sa_attend_noalloc": (_I, [_P, _P, _P, _P, _I, _P, _P, _P]),
    "sa_debug_exp2": (_I, [_I, _P, _P, _I, _P]),
    "sa_attend_sparse": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P]),
    "sa_block_grid": (_I, [_CFGP, ctypes.c_int32, _I32P, _I32P]),
    "sa_debug_attend_stalled": (_I, [_P, _P, _P, _P, _I, _P, _P]),
    "sa_chunk_count": (_I, [_P, _I]),
    "sa_debug_inject_cuda_error": (_I, [_P]),
    "sa_debug_kernel_clock": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
    "sa_debug_layout": (_I, [_P, _I, _I32P, _I32P, _I]),
    "sa_plan": (_I, [_CFGP, ctypes.c_int32, _I32P, _I32P, _I32P, _I]),
    "sa_stream_plan": (_I, [_P, _I, _I, _I32P, _I32P, _I32P, _I]),
    "sa_slot_of": (_I, [_CFGP, ctypes.c_int32]),
    "sa_exchange_block_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "sa_exchange_pack": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "sa_exchange_unpack": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "sa_exchange_pack_to": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_P), _P]),
    "sa_ipc_alloc": (_I, [ctypes.c_size_t, ctypes.POINTER(_P)]),
    "sa_ipc_free": (_I, [_P]),
    "sa_ipc_handle": (_I, [_P, ctypes.c_char_p]),
    "sa_ipc_open": (_I, [ctypes.c_char_p, ctypes.POINTER(_P)]),
    "sa_ipc_close": (_I, [_P]),
    "sa_get_status": (_I, [_P, _P]),
    "sa_last_error": (ctypes.c_char_p, [_P]),
    "sa_status_string": (ctypes.c_char_p, [_I]),
    "sa_build_info": (_I, []),
}


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_causal_streaming_sa_b200.build` (there is no fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype, fn.argtypes = res, args
        _lib = handle
    return _lib


def header_symbols():
    """Entry points declared in include/sa.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SA_API\s+[\w\s\*]+?\b(sa_\w+)\s*\(", text)))


def status_name(status):
    return lib().sa_status_string(int(status)).decode()


def last_error(handle=None):
    return lib().sa_last_error(handle).decode()


def _check(status, handle=None):
    if status != SA_OK:
        raise SaError(status, last_error(handle))


def make_config(batch, heads, head_dim, frames_per_chunk, tok_h, tok_w, sink_chunks,
                window_chunks, softmax_scale=0.0, rope_theta=0.0, ref_frames=0):
    return SaConfig(batch, heads, head_dim, frames_per_chunk, tok_h, tok_w, sink_chunks,
                    window_chunks, softmax_scale, rope_theta, ref_frames)


def sa_validate_config(cfg):
    return lib().sa_validate_config(ctypes.byref(cfg))


def sa_required_bytes(cfg):
    return lib().sa_required_bytes(ctypes.byref(cfg))


def sa_create(cfg, dev_buf, nbytes):
    out = _P()
    _check(lib().sa_create(ctypes.byref(cfg), _P(dev_buf), nbytes, ctypes.byref(out)))
    return out


def sa_destroy(handle):
    _check(lib().sa_destroy(handle))


def sa_reset(handle):
    _check(lib().sa_reset(handle), handle)


def sa_append_chunk(handle, tier, K, V, stream=0):
    _check(lib().sa_append_chunk(handle, tier, _P(K), _P(V), _P(stream)), handle)


def sa_append_chunk_frames(handle, tier, K, V, n_frames, stream=0):
    _check(lib().sa_append_chunk_frames(handle, tier, _P(K), _P(V), int(n_frames), _P(stream)),
           handle)


def sa_set_reference(handle, K, V, stream=0):
    """Set / replace the reference image (K = V = 0 clears it)."""
    _check(lib().sa_set_reference(handle, _P(K or None), _P(V or None), _P(stream)), handle)


def sa_attend_frames(handle, Q, Kc, Vc, n_frames, step_is_final, O, lse=0, stream=0):
    _check(lib().sa_attend_frames(handle, _P(Q), _P(Kc), _P(Vc), int(n_frames),
                                  int(bool(step_is_final)), _P(O), _P(lse or None), _P(stream)),
           handle)


def sa_attend_aligned(handle, Q, Kc, Vc, Ks, Vs, n_frames, step_is_final, O, lse=0, stream=0):
    """Frame-aligned editing attention: the usual keys plus the same-frame source tokens."""
    _check(lib().sa_attend_aligned(handle, _P(Q), _P(Kc), _P(Vc), _P(Ks), _P(Vs), int(n_frames),
                                   int(bool(step_is_final)), _P(O), _P(lse or None), _P(stream)),
           handle)


def sa_stage_keys_frames(handle, Kc, n_frames, stream=0):
    _check(lib().sa_stage_keys_frames(handle, _P(Kc), int(n_frames), _P(stream)), handle)


def sa_attend(handle, Q, Kc, Vc, step_is_final, O, lse=0, stream=0):
    _check(lib().sa_attend(handle, _P(Q), _P(Kc), _P(Vc), int(bool(step_is_final)), _P(O),
                           _P(lse or None), _P(stream)), handle)


def sa_stage_keys(handle, Kc, stream=0):
    _check(lib().sa_stage_keys(handle, _P(Kc), _P(stream)), handle)


def sa_attend_staged(handle, Q, Vc, step_is_final, O, lse=0, stream=0):
    _check(lib().sa_attend_staged(handle, _P(Q), _P(Vc), int(bool(step_is_final)), _P(O),
                                  _P(lse or None), _P(stream)), handle)


def sa_debug_attend_simt(handle, Q, Kc, Vc, step_is_final, O, lse=0, stream=0):
    _check(lib().sa_debug_attend_simt(handle, _P(Q), _P(Kc), _P(Vc), int(bool(step_is_final)),
                                      _P(O), _P(lse or None), _P(stream)), handle)


def sa_attend_noalloc(handle, Q, Kc, Vc, step_is_final, O, lse=0, stream=0):
    """sa_attend that allocates nothing: its key scratch is a fixed array inside
    the library (for callers that cannot allocate device memory)."""
    _check(lib().sa_attend_noalloc(handle, _P(Q), _P(Kc), _P(Vc), int(bool(step_is_final)),
                                   _P(O), _P(lse or None), _P(stream)), handle)


def sa_attend_sparse(handle, Q, Kc, Vc, step_is_final, block_mask, O, lse=0, stream=0):
    _check(lib().sa_attend_sparse(handle, _P(Q), _P(Kc), _P(Vc), int(bool(step_is_final)),
                                  _P(block_mask), _P(O), _P(lse or None), _P(stream)), handle)


def sa_block_grid(cfg, chunk):
    nq, nk = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().sa_block_grid(ctypes.byref(cfg), chunk, ctypes.byref(nq), ctypes.byref(nk)))
    return nq.value, nk.value


def sa_debug_attend_stalled(handle, Q, Kc, Vc, step_is_final, O, stream=0):
    _check(lib().sa_debug_attend_stalled(handle, _P(Q), _P(Kc), _P(Vc), int(bool(step_is_final)),
                                         _P(O), _P(stream)), handle)


def sa_debug_exp2(use_polynomial, x, y, n, stream=0):
    _check(lib().sa_debug_exp2(int(bool(use_polynomial)), _P(x), _P(y), int(n), _P(stream)))


def sa_debug_inject_cuda_error(handle):
    """Make the handle's next launching call fail with SA_ERR_CUDA (test hook)."""
    _check(lib().sa_debug_inject_cuda_error(handle), handle)


def sa_chunk_count(handle, tier):
    return lib().sa_chunk_count(handle, tier)


def sa_debug_kernel_clock():
    """(SM MHz, span in us) of the most recent attention kernel on the current
    device: the median over its CTAs of SM cycles per global-timer nanosecond,
    and first CTA start to last CTA end. Synchronizes the device."""
    mhz, span = ctypes.c_double(), ctypes.c_double()
    _check(lib().sa_debug_kernel_clock(ctypes.byref(mhz), ctypes.byref(span)))
    return mhz.value, span.value


def sa_debug_layout(handle, tier, n):
    """(chunk id per slot, rank per slot) of one tier; -1 marks an empty slot."""
    ids, ranks = (ctypes.c_int32 * n)(), (ctypes.c_int32 * n)()
    m = lib().sa_debug_layout(handle, tier, ids, ranks, n)
    if m < 0:
        raise SaError(-m, last_error(handle))
    return list(ids[:m]), list(ranks[:m])


def sa_plan(cfg, chunk):
    """(ids, slots, t_base) of chunk `chunk`'s attention, computed by the library."""
    cap = SA_MAX_ATTENDED
    ids, slots, tb = ((ctypes.c_int32 * cap)() for _ in range(3))
    n = lib().sa_plan(ctypes.byref(cfg), chunk, ids, slots, tb, cap)
    if n < 0:
        raise SaError(-n, last_error())
    return list(ids[:n]), list(slots[:n]), list(tb[:n])


def sa_stream_plan(handle, step_is_final, n_frames):
    """(ids, t_base, lens) of the plan the handle would run now for a generating
    chunk of n_frames frames (the reference image is not listed)."""
    cap = SA_MAX_ATTENDED
    ids, tb, lens = ((ctypes.c_int32 * cap)() for _ in range(3))
    n = lib().sa_stream_plan(handle, int(bool(step_is_final)), int(n_frames), ids, tb, lens, cap)
    if n < 0:
        raise SaError(-n, last_error(handle))
    return list(ids[:n]), list(tb[:n]), list(lens[:n])


def sa_slot_of(cfg, chunk):
    return lib().sa_slot_of(ctypes.byref(cfg), chunk)


def sa_get_status(handle, stream=0):
    return lib().sa_get_status(handle, _P(stream))


def sa_build_info():
    """Build flags of the loaded library (SA_BUILD_DEVICE_CHECKS: the checked build)."""
    return lib().sa_build_info()


def sa_exchange_block_bytes(B, T, C, D, G, split_dim, payload=SA_PAYLOAD_FP8):
    """Bytes of one destination block of an exchange (0 if the shape is invalid)."""
    return lib().sa_exchange_block_bytes(B, T, C, D, G, split_dim, payload)


def sa_exchange_pack(x, B, T, C, D, G, split_dim, payload, buf, stream=0):
    _check(lib().sa_exchange_pack(_P(x), B, T, C, D, G, split_dim, payload, _P(buf), _P(stream)))


def sa_exchange_unpack(buf, B, T, C, D, G, split_dim, payload, y, stream=0):
    _check(lib().sa_exchange_unpack(_P(buf), B, T, C, D, G, split_dim, payload, _P(y),
                                    _P(stream)))


def sa_exchange_pack_to(x, B, T, C, D, G, split_dim, payload, dst_blocks, stream=0):
    """Pack with block g written straight to device address dst_blocks[g]."""
    arr = (_P * G)(*[_P(int(a)) for a in dst_blocks])
    _check(lib().sa_exchange_pack_to(_P(x), B, T, C, D, G, split_dim, payload, arr, _P(stream)))


def sa_ipc_handle(dev_ptr):
    """The CUDA IPC handle (bytes) of the allocation starting at dev_ptr."""
    buf = ctypes.create_string_buffer(SA_IPC_HANDLE_BYTES)
    _check(lib().sa_ipc_handle(_P(dev_ptr), buf))
    return buf.raw


def sa_ipc_open(handle):
    """Map another process's allocation; returns its device address here."""
    out = _P()
    _check(lib().sa_ipc_open(bytes(handle), ctypes.byref(out)))
    return out.value


def sa_ipc_close(dev_ptr):
    _check(lib().sa_ipc_close(_P(dev_ptr)))


def sa_ipc_alloc(nbytes):
    """A whole device allocation that can be shared by CUDA IPC; returns its address."""
    out = _P()
    _check(lib().sa_ipc_alloc(nbytes, ctypes.byref(out)))
    return out.value


def sa_ipc_free(dev_ptr):
    _check(lib().sa_ipc_free(_P(dev_ptr)))
