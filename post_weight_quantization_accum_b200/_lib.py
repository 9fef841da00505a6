"""ctypes binding of libgptq_b200.so (the C ABI in include/gptq.h).

Argument marshalling only: each function turns torch tensors into device
pointers, passes the current CUDA stream and raises GptqError on a non-OK
status.  Every computation happens in the library's CUDA kernels.  There is no
fallback: if the shared library is missing or fails to load, importing this
module raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgptq_b200.so")

STATUS = {
    0: "GPTQ_OK",
    1: "GPTQ_ERR_INVALID_ARG",
    2: "GPTQ_ERR_NOT_PD",
    3: "GPTQ_ERR_NONFINITE",
    4: "GPTQ_ERR_CUDA",
    5: "GPTQ_ERR_UNSUPPORTED",
    6: "GPTQ_ERR_TIMEOUT",
}
GPTQ_F32, GPTQ_BF16 = 0, 1

# name -> (restype, argtypes); mirrors include/gptq.h
_P = ctypes.c_void_p
_SIGS = {
    "gptq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gptq_version": (ctypes.c_int32, []),
    "gptq_kernel_launches": (ctypes.c_uint64, []),
    "gptq_get_device_status": (ctypes.c_int, [_P]),
    "gptq_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "gptq_set_column_loop": (None, [ctypes.c_int32]),
    "gptq_get_column_loop": (ctypes.c_int32, []),
    "gptq_trace_enable": (None, [ctypes.c_int32]),
    "gptq_trace_read": (ctypes.c_int32, [_P, ctypes.c_int32]),
    "gptq_hessian_workspace_size": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int64]),
    "gptq_hessian_accum": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64,
                                          ctypes.c_float, _P, ctypes.c_size_t, _P]),
    "gptq_prepare_workspace_size": (ctypes.c_size_t, [ctypes.c_int32]),
    "gptq_prepare_hinv": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.c_float, ctypes.c_int32, _P, _P, _P,
                                         _P, ctypes.c_size_t, _P]),
    "gptq_quantize_workspace_size": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]),
    "gptq_num_groups": (ctypes.c_int32, [ctypes.c_int32, ctypes.c_int32]),
    "gptq_quantize_layer": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int64, ctypes.c_int32, _P, _P, _P,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P, _P,
                                           _P, _P, ctypes.c_size_t, _P]),
    "gptq_quantize_rtn": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.c_int32, _P, _P, _P, _P]),
    "gptq_packed_words_per_row": (ctypes.c_int32, [ctypes.c_int32, ctypes.c_int32]),
    "gptq_pack": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P]),
    "gptq_matvec_workspace_size": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int]),
    "gptq_dequant_matvec": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, _P, ctypes.c_int, ctypes.c_int32, _P, _P,
                                           ctypes.c_size_t, _P]),
    "gptq2d_workspace_size": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "gptq2d_round": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _P, _P, ctypes.c_float,
                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t,
                                    _P]),
}


class TraceEntry(ctypes.Structure):
    """gptq_trace_entry: one kernel's launches and summed device milliseconds."""
    _fields_ = [("name", ctypes.c_char * 64), ("launches", ctypes.c_uint64), ("ms", ctypes.c_double)]


class GptqError(RuntimeError):
    """A library call returned a status other than GPTQ_OK."""

    def __init__(self, func, code):
        self.code = code
        self.status = STATUS.get(code, str(code))
        super().__init__(f"{func}: {self.status}")


def load(path=LIB_PATH):
    """Load the shared library and attach the C signatures (raises if absent)."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m post_weight_quantization_accum_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = load()


def check(func, code):
    if code != 0:
        raise GptqError(func, code)
