"""Host-side pieces of the benchmark (CPU): every workload builds with the advertised sizes,
and the algorithmic byte counts match the layer description's format."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("name,batch", [("tiny", 1), ("qproj", 1), ("qproj", 4), ("downproj", 1), ("smollm", 1),
                                        ("vlen4", 1), ("vlen6", 1), ("vlen8", 1), ("vlen12", 1), ("qproj_sym", 1),
                                        ("qproj_groups", 1), ("smollm_vsr", 1)])
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


def test_vsr_and_symmetric_workloads_store_fewer_bytes():
    """The VSR workload keeps its 2% salient weights as whole sub-vectors: 20 bytes per block of 8
    against 48 for the same eight elements in CSR; the symmetric codebook stores a quarter of the
    entries."""
    vs = bench.make_workload("smollm_vsr", 1)
    nb = sum(L.vsr_nblocks for L in vs.layers)
    assert nb > 0 and all(L.nnz == 0 for L in vs.layers)
    vsr_bytes = sum(L.abi_bytes()["vsr"] for L in vs.layers)
    csr_bytes = sum(8 * L.vsr_nblocks * 6 + 4 * (L.n_out + 1) for L in vs.layers)
    assert vsr_bytes < 0.45 * csr_bytes
    q = bench.make_workload("qproj", 1).layers[0]
    qs = bench.make_workload("qproj_sym", 1).layers[0]
    assert qs.abi_bytes()["codebook"] * 4 == q.abi_bytes()["codebook"]


def test_unknown_config_is_rejected():
    with pytest.raises(SystemExit):
        bench.make_workload("nope", 1)


def test_reference_arm_line_carries_the_contract_keys():
    import json
    import subprocess
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    for k in ("metric", "value", "unit", "n_gpus", "ms_per_step", "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert k in d
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["value"] > 0 and d["config"]["workload"].startswith("llama2_7b_qproj")
