"""CPU checks of the C ABI: the library loads, exports every function the header declares, its
size helpers follow the documented layout, and argument validation rejects bad calls before
touching a GPU."""
import ctypes
import os
import re

import pytest

import w4a4_mxfp4_quantized_b200 as mq
from w4a4_mxfp4_quantized_b200 import build as mq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "macaq.h")


@pytest.fixture(scope="module")
def lib():
    mq_build.build()
    return mq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(macaq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("macaq_prep_weights", "macaq_act_quant", "macaq_linear", "macaq_grouped_linear"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    with open(mq.library_path(), "rb") as f:
        assert f.read(4) == b"\x7fELF"


def test_constants_match_the_header():
    """The binding and the tests restate two sizes the header defines: keep them in step."""
    text = open(HEADER).read()
    counters = re.search(r"#define MACAQ_WORKSPACE_COUNTER_BYTES \(\(size_t\)(\d+)\)", text)
    fixed = re.search(r"#define MACAQ_FIXED_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert counters and int(counters.group(1)) == mq.WORKSPACE_COUNTER_BYTES
    import test_zz_no_alloc
    assert fixed and int(fixed.group(1)) << int(fixed.group(2)) == test_zz_no_alloc.FIXED_SCRATCH_BYTES


def test_size_helpers(lib):
    assert mq.sf_bytes(1, 128) == 128 * 4
    assert mq.sf_bytes(128, 4096) == 128 * 128
    assert mq.sf_bytes(129, 4096) == 256 * 128
    assert mq.sf_bytes(0, 4096) == 0
    assert mq.sf_bytes(16, 100) == 0
    assert mq.grouped_sf_bytes(512, 128, 2048) == (4 + 128) * 128 * 64
    assert mq.workspace_bytes(2048, 14336, 4096, 0) >= 0


def test_status_strings(lib):
    for code, name in enumerate(["MACAQ_OK", "MACAQ_ERR_INVALID_ARG", "MACAQ_ERR_SHAPE", "MACAQ_ERR_ALIGNMENT",
                                 "MACAQ_ERR_UNSUPPORTED", "MACAQ_ERR_CUDA", "MACAQ_ERR_TIMEOUT",
                                 "MACAQ_ERR_WORKSPACE"]):
        assert mq.status_str(code) == name
    assert mq.status_str(99) == "MACAQ_ERR_UNKNOWN"


# Validation happens before any CUDA call, so these run without a GPU. Pointers are fake.
P = 0x10000  # 16-byte aligned, never dereferenced


def test_act_quant_rejects_bad_shapes(lib):
    assert lib.macaq_act_quant(P, P, 16, 100, 32, None, 0, P, P, None) == 2      # K % 128
    assert lib.macaq_act_quant(P, P, -1, 256, 32, None, 0, P, P, None) == 2      # M < 0
    assert lib.macaq_act_quant(P, P, 16, 256, 8, None, 0, P, P, None) == 4       # had_block
    assert lib.macaq_act_quant(P, P, 16, 256, 48, None, 0, P, P, None) == 4
    assert lib.macaq_act_quant(P, P, 16, 256, 32, P, 0, P, P, None) == 2         # E < 1 with offsets
    assert lib.macaq_act_quant(None, P, 16, 256, 32, None, 0, P, P, None) == 1   # NULL input
    assert lib.macaq_act_quant(P + 4, P, 16, 256, 32, None, 0, P, P, None) == 3  # misaligned X
    assert lib.macaq_act_quant(P, P, 16, 256, 32, None, 0, P, P + 8, None) == 3  # misaligned SF
    assert lib.macaq_act_quant(P, P, 0, 256, 32, None, 0, P, P, None) == 0       # M == 0: no-op


def test_prep_and_linear_reject_bad_shapes(lib):
    assert lib.macaq_prep_weights(P, P, 100, 256, 32, P, P, P, None) == 2         # N % 128
    assert lib.macaq_linear(0, P, P, None, 16, 200, 256, 32, P, P, P, 0, None, 0, None) == 2   # N % 128
    assert lib.macaq_linear(0, P, P, None, 16, 256, 200, 32, P, P, P, 0, None, 0, None) == 2   # K % 128
    assert lib.macaq_linear(0, P, P, None, 16, 256, 256, 32, P, P, P, 7, None, 0, None) == 1   # out dtype
    assert lib.macaq_linear(5, P, P, None, 16, 256, 256, 32, P, P, P, 0, None, 0, None) == 1   # mode
    assert lib.macaq_linear(0, P, None, None, 16, 256, 256, 32, P, P, P, 0, None, 0, None) == 1
    assert lib.macaq_linear(0, P, P, None, 16, 256, 256, 32, P + 8, P, P, 0, None, 0, None) == 3
    assert lib.macaq_linear(0, P, P, None, 0, 256, 256, 32, P, P, P, 0, None, 0, None) == 0    # M == 0
    assert lib.macaq_grouped_linear(0, P, P, None, None, 4, 16, 256, 256, 32, P, P, P, 0, None, 0, None) == 1
    assert lib.macaq_grouped_linear(0, P, P, None, P, 0, 16, 256, 256, 32, P, P, P, 0, None, 0, None) == 2


def test_fused_mode_rejects_bad_arguments(lib):
    # mode 1 = MACAQ_A_BF16_FUSED: bf16 X in, inv_s, had_block; checked before any CUDA call
    args = lambda **kw: [kw.get(k, d) for k, d in (
        ("mode", 1), ("A", P), ("Asf", None), ("inv", P), ("M", 16), ("N", 256), ("K", 256), ("b", 32), ("Wq", P),
        ("Wsf", P), ("Y", P), ("out", 0), ("ws", P), ("wsb", 1 << 20), ("st", None))]
    assert lib.macaq_linear(*args(b=3)) == 4           # Hadamard block outside {1, 16, 32, 64, 128}
    assert lib.macaq_linear(*args(K=200)) == 2         # K % 128
    assert lib.macaq_linear(*args(out=7)) == 1         # out dtype
    assert lib.macaq_linear(*args(A=None)) == 1        # NULL X
    assert lib.macaq_linear(*args(A=P + 4)) == 3       # misaligned X
    assert lib.macaq_linear(*args(ws=P + 8)) == 3      # misaligned workspace
    assert lib.macaq_linear(*args(M=0)) == 0           # M == 0: no-op
    assert lib.macaq_linear_fixed_scratch(1, P, None, P, 16, 256, 256, 32, P, P, P, 0, None) == 4
    # mode 2 = MACAQ_A_BF16_ONE_LAUNCH: the same arguments and checks
    assert lib.macaq_linear(*args(mode=2, b=3)) == 4
    assert lib.macaq_linear(*args(mode=2, K=200)) == 2
    assert lib.macaq_linear(*args(mode=2, A=P + 4)) == 3
    assert lib.macaq_linear(*args(mode=2, M=0)) == 0
    assert lib.macaq_linear(*args(mode=3)) == 1        # no such mode
    assert lib.macaq_linear_fixed_scratch(2, P, None, P, 16, 256, 256, 32, P, P, P, 0, None) == 4
    assert mq.A_BF16_ONE_LAUNCH == 2
    g = lambda off, E: lib.macaq_grouped_linear(1, P, None, P, off, E, 16, 256, 256, 32, P, P, P, 0, P, 1 << 20, None)
    assert g(None, 4) == 1                             # grouped needs offsets
    assert g(P, 0) == 2                                # E < 1
    assert mq.fused_workspace_bytes(-1, 256, 256) == 0
    assert mq.fused_workspace_bytes(16, 200, 256) == 0


def test_binding_requires_built_library(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(mq, "_lib", None)
    monkeypatch.setattr(mq, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mq.lib()


def test_host_offsets_check(lib):
    """Grouped offsets that the device would clamp are rejected on the host (no GPU needed)."""
    import numpy as np

    mq.check_group_offsets([0, 5, 5, 140, 300], 300)                  # valid, with an empty expert
    mq.check_group_offsets(np.array([0, 0], np.int32), 0)             # one empty expert, no rows
    for bad, rows in [([1, 5, 300], 300),                              # does not start at 0
                      ([0, 5, 299], 300),                              # does not end at total_rows
                      ([0, 7, 5, 300], 300),                           # decreasing
                      ([0, -3, 300], 300),                             # negative
                      ([0, 400, 300], 300)]:                           # past the end, then back
        with pytest.raises(mq.MacaqError, match="MACAQ_ERR_SHAPE"):
            mq.check_group_offsets(bad, rows)
    with pytest.raises(mq.MacaqError, match="MACAQ_ERR_SHAPE"):
        mq.check_group_offsets([0], 0)                                 # E = 0
    assert lib.macaq_check_group_offsets(None, 4, 10) == 1
    big = np.zeros(16386, np.int32)
    assert lib.macaq_check_group_offsets(big.ctypes.data, 16385, 0) == 2   # E above 16384
