"""The bounds-checked build (-DMSA_DEBUG_BOUNDS, libmsa_debug.so) compiles,
loads without a GPU, says what it is and exports the same C ABI as libmsa.so.

Its kernels compare every index they derive from device data with the extent
of its buffer before the access and report MSA_DEV_BOUNDS instead of
faulting; tests/test_gpu_debug_bounds.py runs parity cases and two
precondition violations through it on the GPU."""
import os
import subprocess
import sys

import block_sparse_gqa_mean_b200 as msa
from block_sparse_gqa_mean_b200 import build as libbuild
from test_abi import HEADER, declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROBE = r"""
import ctypes, sys
lib = ctypes.CDLL(sys.argv[1])
names = sys.argv[2].split(",")
missing = [n for n in names if not hasattr(lib, n)]
lib.msa_build_flags.restype = ctypes.c_int32
print(lib.msa_build_flags(), ",".join(missing))
"""


def _probe(path):
    """(build flags, missing symbols) of the library at path, in a fresh
    process so that the two builds never share one."""
    r = subprocess.run([sys.executable, "-c", PROBE, path, ",".join(declared_functions())],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    flags, missing = r.stdout.split()[0], r.stdout.split()[1:]
    return int(flags), missing


def test_header_declares_the_bounds_bit_and_the_build_query():
    text = open(HEADER).read()
    assert "#define MSA_DEV_BOUNDS 0x10u" in text
    assert "#define MSA_BUILD_DEBUG_BOUNDS 0x1" in text
    assert "msa_build_flags" in declared_functions()
    assert msa.MSA_DEV_BOUNDS == 0x10 and msa.MSA_BUILD_DEBUG_BOUNDS == 1


def test_debug_build_compiles_loads_and_reports_itself():
    path = libbuild.build(debug_bounds=True)  # incremental: only stale objects are rebuilt
    assert path == msa.DEBUG_LIB_PATH and os.path.exists(path)
    flags, missing = _probe(path)
    assert flags == msa.MSA_BUILD_DEBUG_BOUNDS
    assert missing == []


def test_regular_build_has_no_checks():
    flags, missing = _probe(libbuild.LIB)
    assert flags == 0
    assert missing == []


def test_every_kernel_source_uses_the_checks():
    """The sources whose kernels derive indices from device data carry checks."""
    csrc = os.path.join(ROOT, "block_sparse_gqa_mean_b200", "csrc")
    for name in ("append_pool.cu", "attn_simt.cu", "select.cu", "decode_splitk.cu",
                 "prefill_tc.cu", "tokens.cu"):
        text = open(os.path.join(csrc, name)).read()
        assert "MSA_IN_BOUNDS" in text or "MSA_RANGE_OK" in text, name
