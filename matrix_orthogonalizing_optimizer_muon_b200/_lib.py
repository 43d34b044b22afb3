"""ctypes binding of libmuon's C ABI (include/muon.h).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels.  The functions keep the C names; ``load()`` raises if the
shared library has not been built, so nothing can silently fall back to
another implementation.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.environ.get("MUON_LIB_PATH") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmuon.so")

MUON_OK = 0
MUON_ERR_INVALID_ARG = 1
MUON_ERR_SHAPE_MISMATCH = 2
MUON_ERR_UNSUPPORTED = 3
MUON_ERR_NO_MEMORY = 4
MUON_ERR_CUDA = 5
MUON_ERR_NONFINITE = 6
MUON_ERR_TIMEOUT = 7
MUON_ERR_ALIAS = 8
MUON_ERR_NOT_CONVERGED = 9

MUON_DT_BF16 = 0
MUON_DT_FP32 = 1
MUON_NS_BF16 = 0
MUON_NS_FP32 = 1
MUON_INIT_ZERO_MOMENTUM = 0x1
MUON_INIT_FP32_NS = 0x2
MUON_INIT_MAX_WORKSPACE = 0x4
MUON_SCALE_MAX_DIM, MUON_SCALE_HIDDEN, MUON_SCALE_UPDATE_NORM = 0, 1, 2
MUON_NUM_PHASES = 6
MUON_PROFILE_LAUNCHES = 1
MUON_PROFILE_SPANS = 2
PHASE_NAMES = ("momentum_normalise", "gram", "poly", "x_update", "finalize", "newton_schulz")
ENTROPY_NUM_PHASES = 4

EXPORTED = ("muon_hparams_default", "muon_init", "muon_init_ex", "muon_num_waves", "muon_inject_wait_timeout",
            "muon_step", "muon_orthogonalize", "muon_workspace_bytes",
            "muon_get_status", "muon_destroy", "muon_status_string", "muon_profile_enable", "muon_profile_read",
            "muon_orthogonalize_noalloc", "muon_adamw_hparams_default", "muon_adamw_init", "muon_adamw_step",
            "muon_adamw_destroy", "muon_entropy_init", "muon_entropy_compute", "muon_entropy_num_singular_values", "muon_entropy_cluster_size",
            "muon_entropy_get_status", "muon_entropy_profile", "muon_entropy_destroy", "muon_pack_init",
            "muon_pack_run", "muon_pack_destroy")


class muon_param_t(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("G", ctypes.c_void_p), ("M", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("g_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class muon_hparams_t(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("weight_decay", ctypes.c_float), ("momentum", ctypes.c_float),
                ("ns_steps", ctypes.c_int32), ("a", ctypes.c_float), ("b", ctypes.c_float),
                ("c", ctypes.c_float), ("rms_scale", ctypes.c_float), ("nesterov", ctypes.c_int32),
                ("ns_precision", ctypes.c_int32), ("scale_mode", ctypes.c_int32), ("hidden_dim", ctypes.c_float)]


class muon_segment_t(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("numel", ctypes.c_int64),
                ("src_dtype", ctypes.c_int32), ("dst_dtype", ctypes.c_int32)]


class muon_adamw_param_t(ctypes.Structure):
    _fields_ = [("P", ctypes.c_void_p), ("G", ctypes.c_void_p), ("m", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("numel", ctypes.c_int64), ("g_dtype", ctypes.c_int32), ("decay", ctypes.c_int32)]


class muon_adamw_hparams_t(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int32)]


class MuonError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def load() -> ctypes.CDLL:
    """Load libmuon.so (once).  Raises if it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libmuon.so not found at {LIB_PATH}; build it with "
                           "`python -m matrix_orthogonalizing_optimizer_muon_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    lib.muon_hparams_default.argtypes = [ctypes.POINTER(muon_hparams_t)]
    lib.muon_hparams_default.restype = ctypes.c_int
    lib.muon_init.argtypes = [ctypes.POINTER(P), ctypes.POINTER(muon_param_t), ctypes.c_int32, ctypes.c_uint32, P]
    lib.muon_init.restype = ctypes.c_int
    lib.muon_init_ex.argtypes = [ctypes.POINTER(P), ctypes.POINTER(muon_param_t), ctypes.c_int32, ctypes.c_uint32,
                                 ctypes.c_size_t, P]
    lib.muon_init_ex.restype = ctypes.c_int
    lib.muon_num_waves.argtypes = [P]
    lib.muon_num_waves.restype = ctypes.c_int32
    lib.muon_inject_wait_timeout.argtypes = [P, ctypes.c_uint32]
    lib.muon_inject_wait_timeout.restype = ctypes.c_int
    lib.muon_pack_init.argtypes = [ctypes.POINTER(P), ctypes.POINTER(muon_segment_t), ctypes.c_int32, P]
    lib.muon_pack_init.restype = ctypes.c_int
    lib.muon_pack_run.argtypes = [P, P]
    lib.muon_pack_run.restype = ctypes.c_int
    lib.muon_pack_destroy.argtypes = [P]
    lib.muon_pack_destroy.restype = None
    lib.muon_step.argtypes = [P, ctypes.POINTER(muon_param_t), ctypes.c_int32, ctypes.POINTER(muon_hparams_t), P, P]
    lib.muon_step.restype = ctypes.c_int
    lib.muon_orthogonalize.argtypes = [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.POINTER(ctypes.c_float), ctypes.c_int32, P]
    lib.muon_orthogonalize.restype = ctypes.c_int
    lib.muon_workspace_bytes.argtypes = [P]
    lib.muon_workspace_bytes.restype = ctypes.c_size_t
    lib.muon_get_status.argtypes = [P]
    lib.muon_get_status.restype = ctypes.c_int
    lib.muon_destroy.argtypes = [P]
    lib.muon_destroy.restype = None
    lib.muon_status_string.argtypes = [ctypes.c_int]
    lib.muon_status_string.restype = ctypes.c_char_p
    lib.muon_profile_enable.argtypes = [P, ctypes.c_int32]
    lib.muon_profile_enable.restype = ctypes.c_int
    lib.muon_profile_read.argtypes = [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                                      ctypes.POINTER(ctypes.c_int32)]
    lib.muon_profile_read.restype = ctypes.c_int
    lib.muon_orthogonalize_noalloc.argtypes = [P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.POINTER(ctypes.c_float), P]
    lib.muon_orthogonalize_noalloc.restype = ctypes.c_int
    lib.muon_adamw_hparams_default.argtypes = [ctypes.POINTER(muon_adamw_hparams_t)]
    lib.muon_adamw_hparams_default.restype = ctypes.c_int
    lib.muon_adamw_init.argtypes = [ctypes.POINTER(P), ctypes.POINTER(muon_adamw_param_t), ctypes.c_int32,
                                    ctypes.c_uint32, P]
    lib.muon_adamw_init.restype = ctypes.c_int
    lib.muon_adamw_step.argtypes = [P, ctypes.POINTER(muon_adamw_param_t), ctypes.c_int32,
                                    ctypes.POINTER(muon_adamw_hparams_t), P]
    lib.muon_adamw_step.restype = ctypes.c_int
    lib.muon_adamw_destroy.argtypes = [P]
    lib.muon_adamw_destroy.restype = None
    lib.muon_entropy_init.argtypes = [ctypes.POINTER(P), ctypes.POINTER(ctypes.c_int64), ctypes.c_int32, P]
    lib.muon_entropy_init.restype = ctypes.c_int
    lib.muon_entropy_compute.argtypes = [P, ctypes.POINTER(P), ctypes.c_int32, P, P, P]
    lib.muon_entropy_compute.restype = ctypes.c_int
    lib.muon_entropy_num_singular_values.argtypes = [P]
    lib.muon_entropy_num_singular_values.restype = ctypes.c_int64
    lib.muon_entropy_cluster_size.argtypes = [P]
    lib.muon_entropy_cluster_size.restype = ctypes.c_int32
    lib.muon_entropy_get_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
    lib.muon_entropy_get_status.restype = ctypes.c_int
    lib.muon_entropy_profile.argtypes = [P, ctypes.c_int32, ctypes.POINTER(ctypes.c_double)]
    lib.muon_entropy_profile.restype = ctypes.c_int
    lib.muon_entropy_destroy.argtypes = [P]
    lib.muon_entropy_destroy.restype = None
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().muon_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != MUON_OK:
        raise MuonError(status, where)


# ------------------------------------------------------------------ same-name wrappers

def muon_hparams_default() -> muon_hparams_t:
    hp = muon_hparams_t()
    check(load().muon_hparams_default(ctypes.byref(hp)), "muon_hparams_default")
    return hp


def muon_init(params, n: int, flags: int, stream: int) -> ctypes.c_void_p:
    plan = ctypes.c_void_p()
    check(load().muon_init(ctypes.byref(plan), params, int(n), int(flags), ctypes.c_void_p(stream)), "muon_init")
    return plan


def muon_init_ex(params, n: int, flags: int, max_workspace_bytes: int, stream: int) -> ctypes.c_void_p:
    plan = ctypes.c_void_p()
    check(load().muon_init_ex(ctypes.byref(plan), params, int(n), int(flags), int(max_workspace_bytes),
                              ctypes.c_void_p(stream)), "muon_init_ex")
    return plan


def muon_num_waves(plan) -> int:
    return int(load().muon_num_waves(plan))


def muon_pack_init(segs, n: int, stream: int) -> ctypes.c_void_p:
    plan = ctypes.c_void_p()
    check(load().muon_pack_init(ctypes.byref(plan), segs, int(n), ctypes.c_void_p(stream)), "muon_pack_init")
    return plan


def muon_pack_run(plan, stream: int) -> None:
    check(load().muon_pack_run(plan, ctypes.c_void_p(stream)), "muon_pack_run")


def muon_pack_destroy(plan) -> None:
    load().muon_pack_destroy(plan)


def muon_inject_wait_timeout(plan, wait_ns: int) -> None:
    check(load().muon_inject_wait_timeout(plan, int(wait_ns)), "muon_inject_wait_timeout")


def muon_step(plan, params, n: int, hp: muon_hparams_t, update_rms_ptr: int | None, stream: int) -> None:
    check(load().muon_step(plan, params, int(n), ctypes.byref(hp), ctypes.c_void_p(update_rms_ptr or 0),
                           ctypes.c_void_p(stream)), "muon_step")


def muon_orthogonalize(plan, x_ptrs, o_ptrs, n: int, in_dtype: int, ns_steps: int, abc, precision: int,
                       stream: int) -> None:
    abc_arr = (ctypes.c_float * 3)(*[float(v) for v in abc])
    check(load().muon_orthogonalize(plan, x_ptrs, o_ptrs, int(n), int(in_dtype), int(ns_steps), abc_arr,
                                    int(precision), ctypes.c_void_p(stream)), "muon_orthogonalize")


def muon_orthogonalize_noalloc(x_ptr: int, o_ptr: int, rows: int, cols: int, in_dtype: int, ns_steps: int, abc,
                               stream: int) -> None:
    abc_arr = (ctypes.c_float * 3)(*[float(v) for v in abc])
    check(load().muon_orthogonalize_noalloc(ctypes.c_void_p(x_ptr), ctypes.c_void_p(o_ptr), int(rows), int(cols),
                                            int(in_dtype), int(ns_steps), abc_arr, ctypes.c_void_p(stream)),
          "muon_orthogonalize_noalloc")


def muon_workspace_bytes(plan) -> int:
    return int(load().muon_workspace_bytes(plan))


def muon_get_status(plan) -> int:
    return int(load().muon_get_status(plan))


def muon_destroy(plan) -> None:
    load().muon_destroy(plan)


def muon_profile_enable(plan, mode: int) -> None:
    check(load().muon_profile_enable(plan, int(mode)), "muon_profile_enable")


def muon_profile_read(plan):
    ms = (ctypes.c_double * MUON_NUM_PHASES)()
    cnt = (ctypes.c_int64 * MUON_NUM_PHASES)()
    calls = ctypes.c_int32()
    check(load().muon_profile_read(plan, ms, cnt, ctypes.byref(calls)), "muon_profile_read")
    return list(ms), list(cnt), int(calls.value)


def muon_adamw_hparams_default() -> muon_adamw_hparams_t:
    hp = muon_adamw_hparams_t()
    check(load().muon_adamw_hparams_default(ctypes.byref(hp)), "muon_adamw_hparams_default")
    return hp


def muon_adamw_init(params, n: int, flags: int, stream: int) -> ctypes.c_void_p:
    plan = ctypes.c_void_p()
    check(load().muon_adamw_init(ctypes.byref(plan), params, int(n), int(flags), ctypes.c_void_p(stream)),
          "muon_adamw_init")
    return plan


def muon_adamw_step(plan, params, n: int, hp: muon_adamw_hparams_t, stream: int) -> None:
    check(load().muon_adamw_step(plan, params, int(n), ctypes.byref(hp), ctypes.c_void_p(stream)), "muon_adamw_step")


def muon_adamw_destroy(plan) -> None:
    load().muon_adamw_destroy(plan)


def muon_entropy_init(shapes, stream: int) -> ctypes.c_void_p:
    flat = (ctypes.c_int64 * (2 * len(shapes)))(*[int(v) for s in shapes for v in s])
    plan = ctypes.c_void_p()
    check(load().muon_entropy_init(ctypes.byref(plan), flat, len(shapes), ctypes.c_void_p(stream)),
          "muon_entropy_init")
    return plan


def muon_entropy_compute(plan, w_ptrs, n: int, h_ptr: int, sigma_ptr: int | None, stream: int) -> None:
    check(load().muon_entropy_compute(plan, w_ptrs, int(n), ctypes.c_void_p(h_ptr), ctypes.c_void_p(sigma_ptr or 0),
                                      ctypes.c_void_p(stream)), "muon_entropy_compute")


def muon_entropy_num_singular_values(plan) -> int:
    return int(load().muon_entropy_num_singular_values(plan))


def muon_entropy_cluster_size(plan) -> int:
    return int(load().muon_entropy_cluster_size(plan))


def muon_entropy_get_status(plan, n: int):
    """(status code, per matrix 1 if its eigenvalues were computed, 0 if it
    was non-finite) -- synchronising read-and-clear."""
    computed = (ctypes.c_int32 * n)()
    st = int(load().muon_entropy_get_status(plan, computed))
    return st, list(computed)


def muon_entropy_profile(plan, enable: bool, read: bool = False):
    ms = (ctypes.c_double * ENTROPY_NUM_PHASES)()
    check(load().muon_entropy_profile(plan, 1 if enable else 0, ms if read else None), "muon_entropy_profile")
    return list(ms) if read else None


def muon_entropy_destroy(plan) -> None:
    load().muon_entropy_destroy(plan)
