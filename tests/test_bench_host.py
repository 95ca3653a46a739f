"""Host-side rules of bench.py that need no GPU: how many independent layers a
workload's steps rotate over (so that no step finds its weights in L2), the
algorithmic bytes of an expert, and the reported configuration."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from moe_expert_layer_renorm_b200 import inputs  # noqa: E402


def test_bytes_per_expert_counts_codes_scales_and_globals():
    H, I = 2048, 768
    codes = 3 * H * I // 2          # two E2M1 codes per byte
    scales = 3 * H * I // 16        # one E4M3 byte per 16 values
    assert bench.bytes_per_expert(H, I) == codes + scales + 12
    assert bench.gate_up_bytes_per_expert(H, I) == 2 * (H * I // 2 + H * I // 16) + 8


@pytest.mark.parametrize("name", ["decode_T1", "decode_T64", "prefill_zipf_T4096", "wide_decode_T1", "tiny"])
def test_rotation_evicts_l2_between_visits(name):
    w = inputs.WORKLOADS[name]
    R = bench.rotation_layers(w, 1)
    per_step = inputs.expected_distinct_experts(w.T, w.E, w.k) * bench.bytes_per_expert(w.H, w.I)
    assert 1 <= R <= 64
    # between two visits of a layer the other R - 1 layers read about 3x L2, unless capped at 64 layers
    assert (R - 1) * per_step >= 3.0 * bench.L2_BYTES or R == 64
    assert bench.rotation_layers(w, R + 5) == min(64, R + 5)   # a larger request is honoured


def test_workload_config_names_the_workload():
    w = inputs.WORKLOADS["decode_T64"]
    cfg = bench.workload_config(w, 4, 512, 2)
    assert cfg["workload"] == "decode_T64" and cfg["T"] == 64 and cfg["E"] == 128 and cfg["k"] == 8
    assert cfg["parallelism"] == "dp2 (independent batches)" and cfg["layers_rotated"] == 4
    assert "L2" in cfg["l2"]
    # the config is a function of the workload and the run alone, so both arms print the same one
    assert cfg == bench.workload_config(w, 4, 512, 2)


def test_every_workload_family_is_reported():
    names = set(bench.ALL_WORKLOADS)
    assert {"tiny", "decode_T1", "decode_T8", "decode_T32", "decode_T64", "prefill_zipf_T4096", "slots512_T1",
            "slots512_T2048", "slots512_T8192", "wide_T8192"} <= names
    assert all(n in inputs.WORKLOADS for n in names)
    assert bench.SWEEP_WORKLOAD == "wide_decode_T1" and inputs.WIDE_SWEEP_LAYERS == 48
    assert bench.MEDIAN_REPLAYS >= 50


def test_e2e_pipeline_with_no_steps_only_gates_the_copy_streams():
    class S:
        def __init__(self):
            self.waits = []

        def wait_event(self, e):
            self.waits.append(e)

    class E:
        def record(self, s):
            raise AssertionError("nothing to record")

    h2d, comp, d2h = S(), S(), S()
    start = object()
    p = bench.E2EPipeline(2, h2d, comp, d2h, E, None, None, None)
    p.run(0, start_event=start)
    assert h2d.waits == [start] and d2h.waits == [start] and comp.waits == []
