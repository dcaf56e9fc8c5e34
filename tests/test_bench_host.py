"""Host-side pieces of the benchmark (CPU): every workload builds with the advertised sizes,
and the algorithmic byte counts match the layer description's format."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("name,batch", [("tiny", 1), ("qproj", 1), ("qproj", 4), ("downproj", 1), ("smollm", 1),
                                        ("vlen4", 1), ("vlen6", 1), ("vlen8", 1), ("vlen12", 1)])
def test_workloads_build(name, batch):
    wl = bench.make_workload(name, batch)
    assert wl.kind == "gemv"
    assert wl.bytes_per_step() > 0 and wl.flops_per_step() > 0
    for li, B in wl.calls:
        assert B == batch and wl.xs[li].shape[0] >= B


def test_qproj_bytes_match_the_survey_count():
    # 4 MiB of 16-bit indices + 1 MiB codebook + CSR (fp16 value, int32 column, int32 row_ptr)
    # + fp16 row and column scales + fp16 x and y
    wl = bench.make_workload("qproj", 1)
    assert wl.bytes_per_step() == 6298668


def test_unknown_config_is_rejected():
    with pytest.raises(SystemExit):
        bench.make_workload("nope", 1)
