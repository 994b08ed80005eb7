"""The C ABI library loads and exports every declared symbol (CPU only: no compute calls)."""
import ctypes
import os
import re

from hybrid_linear_top_lightning_b200 import lisa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "lisa.h")).read()
    return sorted(set(re.findall(r"LISA_API\s+[\w\s\*]+?\b(lisa_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(lisa.EXPORTS)


def test_library_loads_and_exports_every_symbol():
    lib = lisa.load()
    for name in _declared():
        assert hasattr(lib, name), name
    assert lisa.version().startswith("liblisa")
    assert lisa.status_string(lisa.LISA_ERR_WORKSPACE).startswith("workspace")


def test_host_validation_without_gpu():
    """Argument checks run on the host before any launch, so they work with no GPU."""
    good = lisa.make_dims(8, 1, 16383, 16384, 28, 4, 128, 8, 1, 64, 2048)
    assert lisa.lisa_workspace_size(good, lisa.LISA_OP_DECODE_STEP) > 0
    for field, value in [("H_q", 27), ("M", 0), ("n_past", 16384), ("H_Ik", 2), ("d", 0)]:
        bad = lisa.make_dims(8, 1, 16383, 16384, 28, 4, 128, 8, 1, 64, 2048)
        setattr(bad, field, value)
        n = ctypes.c_size_t(0)
        st = lisa.load().lisa_workspace_size(ctypes.byref(bad), lisa.LISA_OP_DECODE_STEP,
                                             ctypes.byref(n))
        assert st == lisa.LISA_ERR_INVALID_ARG, field
    big = lisa.make_dims(1, 1, 0, 1, 2, 1, 512, 1, 1, 32, 4)
    n = ctypes.c_size_t(0)
    assert lisa.load().lisa_workspace_size(ctypes.byref(big), 0, ctypes.byref(n)) == lisa.LISA_ERR_UNSUPPORTED
    # null pointers are rejected before launch
    st = lisa.load().lisa_gate_fuse(ctypes.byref(good), None, None, None, None, None)
    assert st == lisa.LISA_ERR_INVALID_ARG


def test_every_operation_has_a_workspace_size():
    """Each LISA_OP_* the header declares answers lisa_workspace_size; one past
    the last is rejected."""
    src = open(os.path.join(ROOT, "include", "lisa.h")).read()
    ops = {k: int(v) for k, v in re.findall(r"\b(LISA_OP_\w+)\s*=\s*(\d+)", src)}
    assert ops and sorted(ops.values()) == list(range(len(ops)))
    good = lisa.make_dims(8, 1, 16383, 16384, 28, 4, 128, 8, 1, 64, 2048)
    for name, op in ops.items():
        assert getattr(lisa, name) == op, name
        assert lisa.lisa_workspace_size(good, op) > 0, name
    n = ctypes.c_size_t(0)
    st = lisa.load().lisa_workspace_size(ctypes.byref(good), len(ops), ctypes.byref(n))
    assert st == lisa.LISA_ERR_INVALID_ARG
    st = lisa.load().lisa_gate_channel(ctypes.byref(good), 0, None, None, None, None, None, None,
                                       0, None)
    assert st == lisa.LISA_ERR_INVALID_ARG
