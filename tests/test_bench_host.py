"""bench.py's host-side helpers on CPU: the committed traffic record is used
only while every source file of its kernel is unchanged, the roofline peak
falls back when no measured peaks are present, and the clock sampler's parse
of nvidia-smi lines (median SM clock, throttle reasons that were active)."""
import hashlib
import json
import os

import bench


def _record(root, files, read=100, write=20):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    srcs = {}
    for rel, text in files.items():
        p = os.path.join(root, rel)
        os.makedirs(os.path.dirname(p), exist_ok=True)
        with open(p, "w") as f:
            f.write(text)
        srcs[rel] = hashlib.sha256(text.encode()).hexdigest()
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as f:
        json.dump({"k": {"sources": srcs, "workload_name": "wl", "dram_read_bytes": read,
                         "dram_write_bytes": write}}, f)


def test_traffic_only_while_every_source_is_unchanged(tmp_path):
    root = str(tmp_path)
    _record(root, {"csrc/a.cu": "kernel", "csrc/common.cuh": "helpers"})
    assert bench.profiled_traffic("k", "wl", root) == 120
    assert bench.profiled_traffic("other", "wl", root) is None
    assert bench.profiled_traffic("k", "another_workload", root) is None   # captured on another workload
    with open(os.path.join(root, "csrc", "common.cuh"), "a") as f:
        f.write(" ")                                    # a shared header changed
    assert bench.profiled_traffic("k", "wl", root) is None
    os.remove(os.path.join(root, "csrc", "common.cuh"))
    assert bench.profiled_traffic("k", "wl", root) is None


def test_traffic_record_with_no_sources_is_not_used(tmp_path):
    root = str(tmp_path)
    _record(root, {})
    assert bench.profiled_traffic("k", "wl", root) is None


def test_committed_traffic_record_names_existing_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["attn_kernel<128,true>"]
    assert "query_aware_sparse_tb_b200/csrc/attn.cu" in rec["sources"]
    for rel in rec["sources"]:
        assert os.path.exists(os.path.join(bench.ROOT, rel)), rel
    assert rec["dram_read_bytes"] > 0 and rec["dram_write_bytes"] >= 0
    assert rec["workload_name"] in bench.tb_inputs.WORKLOADS


def test_peak_falls_back_without_measured_peaks(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6532.5}))
    assert bench.measured_peaks() == (6532.5, "measured")


class _FakeSmi:
    def __init__(self, text):
        self.text = text

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def test_clock_parse():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.proc = _FakeSmi("1965, 1965, 700.1, Not Active, Not Active, Not Active, Not Active\n"
                       "1300, 1965, 999.0, Not Active, Not Active, Not Active, Active\n"
                       "1900, 1965, 900.0, Not Active, Not Active, Not Active, Not Active\n"
                       "[N/A], 1965, 1.0, Not Active, Not Active, Not Active, Not Active\n")
    got = cs.stop()
    assert got["sm_mhz"] == 1900 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"] and got["samples"] == 3
    cs.proc = None
    assert cs.stop()["sm_mhz"] is None


def test_cpu_baseline_layers_and_extrapolation():
    w = bench.tb_inputs.WORKLOADS["llama64k"]
    assert bench.sample_layers(w) == [0, 1, 31]
    assert bench.sample_layers(bench.tb_inputs.WORKLOADS["tiny300"]) == [0]
    # per-layer samples: 32 layers of (pred + 15 reuse)/16, the MLP of 8
    # producers once per interval, projection per new row
    layers = [dict(t_pred=1.6, t_reuse=0.0, t_mlp=0.8, proj_s_per_row=0.0),
              dict(t_pred=1.6, t_reuse=0.0, t_mlp=None, proj_s_per_row=0.0)]
    assert abs(bench.per_decode_step_s(w, layers) - (32 * 0.1 + 0.8 * 8 / 16)) < 1e-12
    layers = [dict(t_pred=0.0, t_reuse=0.0, t_mlp=None, proj_s_per_row=1.0)]
    assert bench.per_decode_step_s(w, layers) == 32 * 8


def test_cpu_baseline_runs_and_states_the_host():
    w = bench.tb_inputs.WORKLOADS["tiny300"]
    cb = bench.cpu_baseline(w, budget_s=0.2)
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
    assert cb["host_cores"] == os.cpu_count() and "cpu_model" in cb
    assert "layers [0]" in cb["sample"]
