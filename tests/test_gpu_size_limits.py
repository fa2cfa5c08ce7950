"""The largest shape group of the benchmarked parameter sets in one call:
Qwen2.5-7B's 56 tall 18944 x 3584 matrices, 3.8e9 elements, so element offsets
pass 2^31 (about 70 GB on the device). Checked exactly as the other full-size
groups are (test_gpu_fullsize.py): two steps from a zero state, the first and
last matrix teacher-forced against the oracle, NS through its spectrum."""

import pytest

import test_gpu_fullsize as FS

pytestmark = pytest.mark.gpu


def test_largest_group_step(cuda_lib):
    FS.test_full_size_group_step(cuda_lib, 4, 2, "standard")
