"""The C ABI library loads, exports every symbol include/dspark.h declares, and
answers its pure-host queries and argument checks (no GPU needed)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT
from speculative_decoding_draft_sample_b200 import binding as bn
from speculative_decoding_draft_sample_b200 import build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return bn.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dspark.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dspark_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(bn.SIGNATURES)


def test_version_and_strings(lib):
    assert bn.version() >> 16 == 3
    assert lib.dspark_status_string(0) == b"ok"
    assert b"workspace" in lib.dspark_status_string(-4)


def test_workspace_sizes(lib):
    # draft: status block + (max, sum) per request per 256-entry chunk
    assert bn.workspace_bytes(bn.OP_DRAFT, 256, 5, 129280, 256, bn.BF16) == 256 + 256 * 505 * 8
    # verify: status block, the draft's partials (disjoint, so the target statistics
    # can be made beside the draft), (max, sum) per request, target row and 2 KB
    # chunk of rows 0..K, the work counter, the verification order (4 bytes per request)
    assert bn.workspace_bytes(bn.OP_VERIFY, 256, 5, 129280, 256, bn.BF16) == \
        256 + 256 * 505 * 8 + 256 * 6 * 127 * 8 + 256 + 1024
    assert bn.workspace_bytes(bn.OP_SCHEDULE, 1024, 8, 0, 0, 0) == 256
    assert bn.workspace_bytes(bn.OP_SCHEDULE, 1024, 65, 0, 0, 0) == 0  # K > 64
    assert bn.workspace_bytes(bn.OP_DRAFT, 4, 4, 1001, 16, bn.F32) == 0  # V % 8
    assert bn.workspace_bytes(bn.OP_VERIFY, 4, 65, 1024, 16, bn.F32) == 0  # K > 64
    assert bn.workspace_bytes(9, 4, 4, 1024, 16, bn.F32) == 0
    # calibration: status block, 888 CTAs x 256 fp64 losses, 888 x K x 15 x 3 fp64 bin sums
    assert bn.workspace_bytes(bn.OP_CALIB, 1000, 5, 0, 0, 0) == 256 + 888 * 256 * 8 + 888 * 5 * 15 * 3 * 8
    assert bn.workspace_bytes(bn.OP_CALIB, 1000, 65, 0, 0, 0) == 0


def test_null_pointers_rejected_before_any_device_call(lib):
    p = ctypes.c_void_p(0)
    assert lib.dspark_draft_sample(p, p, p, p, p, p, 4, 4, 1024, 16, 0, 1, 0, p, p, p, p, p, p, 0, p) == -1
    assert lib.dspark_draft_sample_beside(p, p, p, p, p, p, p, 4, 4, 1024, 16, 0, 1, 0, p, p, p, p,
                                          p, p, 20, p, 0, p) == -1
    assert lib.dspark_verify(p, p, p, p, p, p, p, 4, 4, 1024, 0, 1, 0, p, p, p, p, 0, p) == -1
    assert lib.dspark_verify_from_stats(p, p, p, p, p, p, p, 4, 4, 1024, 0, 1, 0, p, p, p, p, 0,
                                        p) == -1
    assert lib.dspark_verify_target_stats(p, p, p, 4, 4, 1024, 0, p, 0, p) == -1
    assert lib.dspark_draft_logits(p, p, p, p, p, p, p, 4, 4, 1024, 16, 0, 1, p, p, 0, p) == -1
    assert lib.dspark_draft_pick(p, p, p, 4, 4, 1024, 0, 1, 0, 1, p, p, p, p, p, 0, p) == -1
    assert lib.dspark_sts_fit(p, p, 100, 5, p, p, p, p, p, 0, p) == -1
    assert lib.dspark_prefix_schedule(p, p, p, 0.0, 4, 4, 0, 0.0, p, p, p, 0, p) == -1
    assert lib.dspark_read_status(p, p, None, None) == -1
    assert lib.dspark_clear_status(p, p) == -1
