"""The benchmark's JSON line on the CPU: the keys and values the contract asks
for, in the decode line (assembled from synthetic measurements) and in the
reference arm (the oracle, run for real on a bounded sample)."""
import ast
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
             "scaling", "vs_baseline", "dtype", "data", "config"}


def _fake_decode_result():
    roofline = {"bound": "hbm", "achieved": 1300.0, "peak": 6546.6, "unit": "GB/s", "frac": 1300.0 / 6546.6,
                "traffic": 15997440}
    return {
        "ms_per_step": 0.8, "units_per_step": 40, "roofline": roofline,
        "roofline_ffn": dict(roofline, frac=0.2), "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
        "e2e": {"value": 47000.0, "unit": "tokens/s", "h2d_bytes_per_step": 163840, "d2h_bytes_per_step": 163840},
        "gpu_launches": 16000, "breakdown_us_per_layer": {"route": 6.0}, "_host_layers": [],
    }


def test_decode_line_has_the_contract_keys():
    peaks = bench.load_peaks()
    res = _fake_decode_result()
    line = bench.decode_line(res, 0.8, 40.0, 1, 200, 10, peaks)
    assert BASE_KEYS <= set(line)
    assert line["value"] == 40.0 / 0.8e-3
    assert line["n_gpus"] == 1 and line["steps"] == 200 and line["warmup"] == 10
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["config"]["workload"] == bench.DECODE_WORKLOAD and "l2" in line["config"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(line["roofline"])
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(line["e2e"])
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(line["clocks"])
    assert line["gpu_launches"] > 0
    json.dumps(line)
    # two replicas: the job's work is both ranks' passes over the slower rank's time
    two = bench.decode_line(res, 0.9, 80.0, 2, 200, 10, peaks)
    assert two["value"] == 80.0 / 0.9e-3 and two["config"]["parallelism"] == "replicas"


def test_run_decode_returns_what_the_line_reads():
    """run_decode (GPU) returns a dict literal; it must carry every key the
    line reads from it."""
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    fn = next(n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name == "run_decode")
    ret = [n for n in ast.walk(fn) if isinstance(n, ast.Return) and isinstance(n.value, ast.Dict)][-1]
    keys = {k.value for k in ret.value.keys}
    line_fn = next(n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name == "decode_line")
    read = {n.slice.value for n in ast.walk(line_fn)
            if isinstance(n, ast.Subscript) and isinstance(n.value, ast.Name) and n.value.id == "res"}
    assert read and read <= keys, read - keys
    assert {"ms_per_step", "units_per_step", "_host_layers"} <= keys


def test_reference_arm_line(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert BASE_KEYS <= set(line)
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.DECODE_WORKLOAD
    assert line["steps"] == 2 and line["value"] > 0
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"] and cpu["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_report_only_workloads():
    """The report-only layers: configurations 0, 2 and 4 as the generator
    defines them, and decode-layer shapes at 2, 4, 8 and 16 tokens."""
    other = bench.other_config_specs()
    assert sorted(other) == ["0", "2", "4"]
    assert [(other[k][0].T, other[k][0].H) for k in ("0", "2", "4")] == [(8, 512), (512, 2048), (16384, 2048)]
    small = bench.small_t_specs()
    assert {k: (s.T, s.H, s.I, s.E) for k, (s, _) in small.items()} == {
        "T2": (2, 2048, 512, 256), "T4": (4, 2048, 512, 256), "T8": (8, 2048, 512, 256), "T16": (16, 2048, 512, 256)}
