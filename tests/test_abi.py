"""The C-ABI library loads, exports every entry point include/dsmoe.h declares, and its
host-only entry points behave as documented. No GPU compute is called here."""
import ctypes
import os
import re

import pytest

import mixture_experts_layer_score_b200 as M
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsmoe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(M.ABI_FUNCTIONS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(M.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings():
    assert M.dsmoe_abi_version() == 1
    names = [M.dsmoe_status_string(i) for i in range(6)]
    assert names[0] == "ok" and len(set(names)) == 6
    assert M.dsmoe_status_string(99) == "unknown status"
    assert M.stage_names() == ["router", "select", "scan", "permute", "gemm_gate_up", "gemm_down", "combine",
                              "shared_experts"]


@pytest.mark.parametrize("name", sorted(W.CONFIGS))
def test_every_workload_config_is_accepted(name):
    c = W.get_config(name)
    cfg = M.cfg_from(c, c.T)
    assert M.dsmoe_check_config(cfg) == M.DSMOE_OK, M.dsmoe_last_error()
    assert M.dsmoe_workspace_bytes(cfg) > 0


def _cfg(**kw):
    base = dict(d_model=256, n_routed=64, top_k=7, d_ff=128, n_shared=1, d_ff_shared=128, max_tokens=512)
    base.update(kw)
    return M.make_cfg(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(d_model=0), M.DSMOE_ERR_INVALID_ARG),
    (dict(top_k=65), M.DSMOE_ERR_INVALID_ARG),
    (dict(top_k=0), M.DSMOE_ERR_INVALID_ARG),
    (dict(score=7), M.DSMOE_ERR_INVALID_ARG),
    (dict(bias_mode=3), M.DSMOE_ERR_INVALID_ARG),
    (dict(renormalize=2), M.DSMOE_ERR_INVALID_ARG),
    (dict(n_shared=1, d_ff_shared=0), M.DSMOE_ERR_INVALID_ARG),
    (dict(max_tokens=0), M.DSMOE_ERR_INVALID_ARG),
    (dict(score=3, top_k=2), M.DSMOE_ERR_INVALID_ARG),
    (dict(score=3, top_k=1, bias_mode=1), M.DSMOE_ERR_INVALID_ARG),
    (dict(score=3, top_k=1, hash_mod=65), M.DSMOE_ERR_INVALID_ARG),
    (dict(d_model=200), M.DSMOE_ERR_UNSUPPORTED),
    (dict(d_ff=96), M.DSMOE_ERR_UNSUPPORTED),
    (dict(n_routed=600, top_k=8), M.DSMOE_ERR_UNSUPPORTED),
    (dict(top_k=17), M.DSMOE_ERR_UNSUPPORTED),
    (dict(n_shared=9), M.DSMOE_ERR_UNSUPPORTED),
])
def test_check_config_rejects(kw, expect):
    st = M.dsmoe_check_config(_cfg(**kw))
    assert st == expect, (kw, st, M.dsmoe_last_error())
    assert M.dsmoe_last_error() != ""


def test_check_config_null():
    lib = ctypes.CDLL(M.LIB_PATH)
    lib.dsmoe_check_config.argtypes = [ctypes.c_void_p]
    assert lib.dsmoe_check_config(None) == M.DSMOE_ERR_INVALID_ARG


def test_workspace_grows_with_tokens():
    a = M.dsmoe_workspace_bytes(_cfg(max_tokens=100))
    b = M.dsmoe_workspace_bytes(_cfg(max_tokens=200))
    assert b > a


def test_null_handle_is_rejected_without_a_gpu():
    lib = ctypes.CDLL(M.LIB_PATH)
    lib.dsmoe_get_status.argtypes = [ctypes.c_void_p]
    assert lib.dsmoe_get_status(None) == M.DSMOE_ERR_INVALID_ARG
    lib.dsmoe_destroy.argtypes = [ctypes.c_void_p]
    lib.dsmoe_destroy(None)  # documented no-op
    with pytest.raises(M.DsmoeError):
        M.dsmoe_set_timing(None, 1)
    with pytest.raises(M.DsmoeError):
        M.dsmoe_set_gemm_kernel(None, M.DSMOE_GEMM_SINGLE)
    assert M.dsmoe_get_gemm_kernel(None) == -1


def test_role_cycle_counters_need_the_profiling_build():
    """The default library carries no role counters: the call says so before touching a GPU;
    a short buffer is rejected first."""
    if os.environ.get("DSMOE_LIBRARY"):
        pytest.skip("a non-default library build is loaded")
    lib = ctypes.CDLL(M.LIB_PATH)
    lib.dsmoe_gemm_role_cycles.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    buf = (ctypes.c_uint64 * 8)()
    assert lib.dsmoe_gemm_role_cycles(buf, 8) == M.DSMOE_ERR_INVALID_ARG
    with pytest.raises(M.DsmoeError) as ei:
        M.dsmoe_gemm_role_cycles()
    assert ei.value.status == M.DSMOE_ERR_UNSUPPORTED
