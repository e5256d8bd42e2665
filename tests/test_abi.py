"""The C-ABI library on a machine without a GPU: it builds for sm_100a,
loads, exports every entry point include/ue.h declares, and rejects bad
arguments on the host before any CUDA work (no compute call is made)."""
import ctypes
import os
import re

import pytest

import token_rerouting_b200 as ue
from token_rerouting_b200 import build as ue_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ue_build.build()
    return ue.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "ue.h")).read()
    return sorted(set(re.findall(r"^ue_status\s+(ue_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(ue.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_symbols_are_c_linkage():
    out = os.popen(f"nm -D --defined-only {ue_build.LIB}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_built_for_sm100a_only():
    out = os.popen(f"cuobjdump --list-elf {ue_build.LIB} 2>/dev/null").read()
    if not out:
        pytest.skip("cuobjdump unavailable")
    arches = set(re.findall(r"sm_(\d+a?)", out))
    assert arches == {"100a"}, arches


BAD_CONFIGS = [
    (0, 4, 8, 2, 1, 8),      # R = 0
    (3, 4, 8, 2, 1, 8),      # E % R != 0
    (2, 4, 8, 9, 1, 8),      # K > E
    (2, 4, 512, 2, 1, 8),    # E > 256
    (2, 4, 8, 2, 9, 8),      # S > 8
    (64, 4, 128, 2, 5, 8),   # R*S > 256
    (2, 0, 8, 2, 1, 8),      # T = 0
    (2, 4, 8, 2, 1, 12),     # d % 8 != 0
    (2, 4, 8, 2, 1, 32768),  # d too large
    (128, 1 << 20, 128, 8, 1, 8),  # Q >= 2^30
]


@pytest.mark.parametrize("cfg", BAD_CONFIGS)
def test_init_rejects_bad_config_before_cuda(lib, cfg):
    h = ctypes.c_void_p(1234)
    rc = lib.ue_init(ctypes.byref(ue.ue_config(*cfg)), 0, ctypes.byref(h))
    assert rc == ue.UE_ERR_INVALID_ARG
    assert h.value is None


def test_init_null_out(lib):
    assert lib.ue_init(ctypes.byref(ue.ue_config(2, 4, 8, 2, 1, 8)), 0, None) == ue.UE_ERR_INVALID_ARG


def test_calls_reject_null_context(lib):
    assert lib.ue_gate_topk(None, 16, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_count(None, 16, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_plan(None, 16, None, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_reroute(None, 16, None, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_plan_reroute(None, 16, 16, None, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    opts = ue.plan_opts(ue.UE_SOLVER_BISECT)
    assert lib.ue_plan_ex(None, 16, ctypes.byref(opts), None, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_reroute_ex(None, 16, None, 1, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_locality_split(None, 16, None, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_reroute_local(None, 16, 16, None, 16, 16, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_permute(None, 16, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_combine(None, 16, 16, 16, 16, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_get_error(None, None) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_debug_set_lookback_limit(None, 5) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_debug_drop_first_publish(None, 1) == ue.UE_ERR_INVALID_ARG
    assert lib.ue_destroy(None) == ue.UE_OK


def test_init_without_gpu_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p(1234)
    rc = lib.ue_init(ctypes.byref(ue.ue_config(8, 512, 64, 4, 2, 256)), 0, ctypes.byref(h))
    assert rc in (ue.UE_ERR_CUDA, ue.UE_ERR_INVALID_ARG)
    assert h.value is None


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not found"):
        ue.load_library(str(tmp_path / "libue.so"))


def test_header_documents_every_entry_point():
    """Every entry point ue.h declares sits under a comment that states its
    error behaviour (an error code, or errors "as for" another call) and
    names its source on the pages, or says that the pages have none."""
    text = open(os.path.join(ROOT, "include", "ue.h")).read()
    for name in ue.EXPORTS:
        m = re.search(r"ue_status\s+" + name + r"\s*\(", text)
        assert m, name
        end = text.rfind("*/", 0, m.start())
        start = text.rfind("/*", 0, end)
        between = text[end + 2:m.start()]
        # only other prototypes may stand between the comment and this one
        assert re.fullmatch(r"(\s|ue_status\s+\w+\s*\([^;]*\);)*", between), name
        doc = text[start:end]
        assert re.search(r"UE_ERR|[Ee]rrors?\b", doc), f"{name}: no error behaviour"
        assert re.search(r'"[A-Z][^"]+"|README|no counterpart', doc), f"{name}: no source"
