"""Host logic of bench.py that decides what the JSON line reports, on CPU.

* ``roofline.traffic`` comes from a committed ncu summary only while the
  kernel sources it was taken on are unchanged: the summary's source hash
  must match, else the field is null.
* The roofline denominator is the measured copy bandwidth when the
  measured-peaks file is there, else the fallback figure.
* Every committed summary that bench.py reads parses and names a traffic
  figure."""
import json
import os

import pytest

import bench


def fake_root(tmp_path, sources):
    csrc = tmp_path / "lossless_bf16_kv_splitzip_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, body in sources.items():
        (csrc / name).write_bytes(body)
    (tmp_path / "profiles").mkdir()
    return tmp_path


def write_profile(root, name, sha, traffic):
    (root / "profiles" / name).write_text(
        "# decode_kernel -- test summary\n\n"
        "| counter | value |\n|---|---|\n| dram__bytes_read.sum | 1 |\n\n"
        f"traffic_per_full_launch_bytes: {traffic}\n"
        f"kernel_source_sha256: {sha}  (sz_decode.cu + sz_internal.cuh)\n")


SOURCES = {"sz_decode.cu": b"decode v1\n", "sz_internal.cuh": b"common v1\n", "sz_encode.cu": b"enc\n"}


def test_hash_of_tree_equals_hash_of_files(tmp_path, monkeypatch):
    root = fake_root(tmp_path, SOURCES)
    monkeypatch.setattr(bench, "ROOT", str(root))
    files = ("sz_decode.cu", "sz_internal.cuh")
    assert bench.kernel_source_hash(files) == bench.kernel_source_hash(files, tree=SOURCES)
    # the order of the names does not matter, the content does
    assert bench.kernel_source_hash(files[::-1]) == bench.kernel_source_hash(files)
    other = dict(SOURCES, **{"sz_decode.cu": b"decode v2\n"})
    assert bench.kernel_source_hash(files, tree=other) != bench.kernel_source_hash(files)
    # a file outside the set does not move the hash
    other = dict(SOURCES, **{"sz_encode.cu": b"enc v2\n"})
    assert bench.kernel_source_hash(files, tree=other) == bench.kernel_source_hash(files)


def test_traffic_is_scaled_while_sources_match(tmp_path, monkeypatch):
    root = fake_root(tmp_path, SOURCES)
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_hash(bench.PROFILE_SOURCES["decode"])
    write_profile(root, bench.PROFILE_FILES["decode"], sha, 8_000_000_000)
    assert bench.profiled_traffic("decode", 64, 64) == 8_000_000_000
    assert bench.profiled_traffic("decode", 16, 64) == 2_000_000_000


def test_traffic_is_null_once_a_source_changed(tmp_path, monkeypatch):
    root = fake_root(tmp_path, SOURCES)
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_hash(bench.PROFILE_SOURCES["decode"])
    write_profile(root, bench.PROFILE_FILES["decode"], sha, 8_000_000_000)
    (root / "lossless_bf16_kv_splitzip_b200" / "csrc" / "sz_internal.cuh").write_bytes(b"common v2\n")
    assert bench.profiled_traffic("decode", 64, 64) is None


@pytest.mark.parametrize("body", ["", "traffic_per_full_launch_bytes: 12\n",
                                  "kernel_source_sha256: 0000000000000000\ntraffic_per_full_launch_bytes: x\n"])
def test_traffic_is_null_for_a_bad_summary(tmp_path, monkeypatch, body):
    root = fake_root(tmp_path, SOURCES)
    monkeypatch.setattr(bench, "ROOT", str(root))
    (root / "profiles" / bench.PROFILE_FILES["decode"]).write_text(body)
    assert bench.profiled_traffic("decode", 64, 64) is None


def test_traffic_is_null_without_a_summary(tmp_path, monkeypatch):
    root = fake_root(tmp_path, SOURCES)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.profiled_traffic("decode", 64, 64) is None
    assert bench.profiled_traffic("no such phase", 64, 64) is None


def test_peak_from_the_measured_file_else_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6457.1, "bf16_tflops": 1590}))
    assert bench.measured_peak() == (6457.1, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    assert bench.FALLBACK_HBM_GBS < bench.SPEC_HBM_GBS


@pytest.mark.parametrize("phase", sorted(bench.PROFILE_FILES))
def test_committed_summaries_parse(phase):
    path = os.path.join(bench.ROOT, "profiles", bench.PROFILE_FILES[phase])
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith(("|", "#", " ")):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    assert int(fields["traffic_per_full_launch_bytes"]) > 0
    sha = fields["kernel_source_sha256"].split(" ")[0]
    assert len(sha) == 16 and int(sha, 16) >= 0


def test_job_config_states_the_spread_over_gpus():
    cfg = {"workload": "llama3-8b-kv-32k", "bytes": 4}
    one = bench.job_config(cfg, 1)
    assert one["parallelism"] == "1 GPU" and one["workload"] == cfg["workload"]
    eight = bench.job_config(cfg, 8)
    assert "replicas x8" in eight["parallelism"] and "each rank codes its own copy" in eight["parallelism"]
    assert "parallelism" not in cfg  # the workload's own config is left as it was


def test_host_facts_name_cores_and_model():
    f = bench.host_facts()
    assert f["host_cores"] == os.cpu_count()
    assert f["cpu_model"] is None or isinstance(f["cpu_model"], str)
