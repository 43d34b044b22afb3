"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, and rejects bad arguments before it
touches the device."""

import ctypes
import os
import re

import pytest

from matrix_orthogonalizing_optimizer_muon_b200 import _lib as L
from matrix_orthogonalizing_optimizer_muon_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_symbols():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        names |= set(re.findall(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", text))
    return names


def test_header_declares_the_entry_points():
    assert declared_symbols() == set(L.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_no_other_exported_functions(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {s for s in exported if s.startswith("muon_")} == declared_symbols()


def test_status_strings(lib):
    for code in range(0, 10):
        assert L.status_string(code) != "unknown status"
    assert L.status_string(0) == "ok"
    assert L.status_string(123) == "unknown status"


def test_default_hparams_are_the_pages_values(lib):
    hp = L.muon_hparams_default()
    assert abs(hp.a - 3.4445) < 1e-6 and abs(hp.b + 4.7750) < 1e-6 and abs(hp.c - 2.0315) < 1e-6
    assert hp.ns_steps == 5 and abs(hp.momentum - 0.95) < 1e-7 and abs(hp.rms_scale - 0.2) < 1e-7
    assert abs(hp.weight_decay - 0.1) < 1e-7 and abs(hp.lr - 4.2e-4) < 1e-10
    assert hp.nesterov == 1 and hp.ns_precision == L.MUON_NS_BF16
    assert hp.scale_mode == L.MUON_SCALE_MAX_DIM and hp.hidden_dim == 0.0
    assert lib.muon_hparams_default(None) == L.MUON_ERR_INVALID_ARG


def test_binding_layouts_and_enums_match_the_header():
    import re
    hdr = open(os.path.join(ROOT, "include", "muon.h")).read()
    # every field of muon_hparams_t is 4 bytes wide, in declaration order
    end = hdr.index("} muon_hparams_t;")
    body = hdr[hdr.rindex("typedef struct {", 0, end) + len("typedef struct {"):end]
    names = re.findall(r"^\s*(?:float|int32_t)\s+([\w, ]+);", body, re.M)
    fields = [n.strip() for group in names for n in group.split(",")]
    assert fields == [f for f, _ in L.muon_hparams_t._fields_]
    assert ctypes.sizeof(L.muon_hparams_t) == 4 * len(fields)
    for name in ("MUON_SCALE_MAX_DIM", "MUON_SCALE_HIDDEN", "MUON_SCALE_UPDATE_NORM", "MUON_NS_BF16", "MUON_NS_FP32"):
        m = re.search(name + r"\s*=\s*(\d+)", hdr)
        assert m and int(m.group(1)) == getattr(L, name), name
    for name in ("MUON_NUM_PHASES", "MUON_PROFILE_LAUNCHES", "MUON_PROFILE_SPANS", "MUON_INIT_ZERO_MOMENTUM",
                 "MUON_INIT_FP32_NS", "MUON_INIT_MAX_WORKSPACE"):
        m = re.search(r"#define\s+" + name + r"\s+(0x[0-9a-fA-F]+|\d+)", hdr)
        assert m and int(m.group(1), 0) == getattr(L, name), name
    assert len(L.PHASE_NAMES) == L.MUON_NUM_PHASES


def test_init_rejects_bad_arguments_before_any_cuda_call(lib):
    plan = ctypes.c_void_p()
    arr = (L.muon_param_t * 2)()
    arr[0].rows, arr[0].cols = 4, 4
    arr[1].rows, arr[1].cols = 4, 4
    assert lib.muon_init(None, arr, 2, 0, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_init(ctypes.byref(plan), None, 2, 0, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_init(ctypes.byref(plan), arr, 0, 0, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_init(ctypes.byref(plan), arr, 2, 0x100, None) == L.MUON_ERR_INVALID_ARG
    arr[1].cols = 0
    assert lib.muon_init(ctypes.byref(plan), arr, 2, 0, None) == L.MUON_ERR_INVALID_ARG
    arr[1].cols = 70000
    assert lib.muon_init(ctypes.byref(plan), arr, 2, 0, None) == L.MUON_ERR_INVALID_ARG
    arr[1].cols = 4
    arr[1].reserved = 1
    assert lib.muon_init(ctypes.byref(plan), arr, 2, 0, None) == L.MUON_ERR_INVALID_ARG
    arr[1].reserved = 0
    # zero-momentum needs every M pointer
    assert lib.muon_init(ctypes.byref(plan), arr, 2, L.MUON_INIT_ZERO_MOMENTUM, None) == L.MUON_ERR_INVALID_ARG
    assert plan.value is None


def test_init_ex_flag_and_budget_must_agree(lib):
    plan = ctypes.c_void_p()
    arr = (L.muon_param_t * 1)()
    arr[0].rows, arr[0].cols = 4, 4
    # the cap flag needs a budget, a budget needs the flag, muon_init takes no cap
    assert lib.muon_init_ex(ctypes.byref(plan), arr, 1, L.MUON_INIT_MAX_WORKSPACE, 0, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_init_ex(ctypes.byref(plan), arr, 1, 0, 1 << 30, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_init(ctypes.byref(plan), arr, 1, L.MUON_INIT_MAX_WORKSPACE, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_init_ex(None, arr, 1, 0, 0, None) == L.MUON_ERR_INVALID_ARG
    assert plan.value is None
    assert lib.muon_num_waves(None) == -1
    m = __import__("re").search(r"MUON_INIT_MAX_WORKSPACE\s+(0x[0-9a-fA-F]+)u",
                                open(os.path.join(ROOT, "include", "muon.h")).read())
    assert m and int(m.group(1), 16) == L.MUON_INIT_MAX_WORKSPACE


def test_pack_init_rejects_bad_segments_before_any_cuda_call(lib):
    plan = ctypes.c_void_p()
    segs = (L.muon_segment_t * 2)()
    segs[0].src, segs[0].dst, segs[0].numel = 0x10000, 0x20000, 100
    segs[1].src, segs[1].dst, segs[1].numel = 0x30000, 0x40000, 100
    assert lib.muon_pack_init(None, segs, 2, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_pack_init(ctypes.byref(plan), None, 2, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_pack_init(ctypes.byref(plan), segs, 0, None) == L.MUON_ERR_INVALID_ARG
    segs[1].dst_dtype = 5
    assert lib.muon_pack_init(ctypes.byref(plan), segs, 2, None) == L.MUON_ERR_INVALID_ARG
    segs[1].dst_dtype = L.MUON_DT_FP32
    segs[1].dst = 0x20000 + 100          # inside the first destination (100 bf16 = 200 bytes)
    assert lib.muon_pack_init(ctypes.byref(plan), segs, 2, None) == L.MUON_ERR_ALIAS
    segs[1].dst = 0x10000 + 8            # over the first source
    assert lib.muon_pack_init(ctypes.byref(plan), segs, 2, None) == L.MUON_ERR_ALIAS
    segs[1].numel = 0
    assert lib.muon_pack_init(ctypes.byref(plan), segs, 2, None) == L.MUON_ERR_INVALID_ARG
    assert plan.value is None
    assert lib.muon_pack_run(None, None) == L.MUON_ERR_INVALID_ARG
    lib.muon_pack_destroy(None)


def test_null_plan_calls(lib):
    hp = L.muon_hparams_default()
    arr = (L.muon_param_t * 1)()
    assert lib.muon_step(None, arr, 1, ctypes.byref(hp), None, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_workspace_bytes(None) == 0
    assert lib.muon_get_status(None) == L.MUON_ERR_INVALID_ARG
    lib.muon_destroy(None)
    abc = (ctypes.c_float * 3)(1, 0, 0)
    assert lib.muon_orthogonalize(None, None, None, 1, 0, 5, abc, 0, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_profile_enable(None, 1) == L.MUON_ERR_INVALID_ARG


def test_entropy_entry_points_reject_bad_arguments_before_any_cuda_call(lib):
    plan = ctypes.c_void_p()
    shapes = (ctypes.c_int64 * 4)(16, 24, 8, 8)
    assert lib.muon_entropy_init(None, shapes, 2, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_entropy_init(ctypes.byref(plan), None, 2, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_entropy_init(ctypes.byref(plan), shapes, 0, None) == L.MUON_ERR_INVALID_ARG
    for bad in ((0, 5), (5, 0), (-1, 4), (1 << 20, 1 << 12)):
        arr = (ctypes.c_int64 * 2)(*bad)
        assert lib.muon_entropy_init(ctypes.byref(plan), arr, 1, None) == L.MUON_ERR_INVALID_ARG, bad
    big = (ctypes.c_int64 * 2)(8193, 8200)
    assert lib.muon_entropy_init(ctypes.byref(plan), big, 1, None) == L.MUON_ERR_UNSUPPORTED
    assert plan.value is None
    assert lib.muon_entropy_compute(None, None, 1, None, None, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_entropy_get_status(None, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_entropy_profile(None, 1, None) == L.MUON_ERR_INVALID_ARG
    assert lib.muon_entropy_num_singular_values(None) == -1
    assert lib.muon_entropy_cluster_size(None) == -1
    lib.muon_entropy_destroy(None)


def test_build_flags_target_sm100a():
    assert "arch=compute_100a,code=sm_100a" in B.ARCH
    assert "-lineinfo" in B.FLAGS
