"""bench.py's reference arm on the CPU: the JSON line it prints (the oracle
timed on a bounded sample of the same workload) and its behaviour on ranks
other than 0 under a multi-rank launch."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, extra_args=()):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "3", *extra_args],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_the_contract_line():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"].startswith("low-bit linear int TOPS")
    assert d["unit"] == "TOPS" and d["value"] > 0 and d["higher_is_better"] is True
    assert (d["steps"], d["warmup"], d["n_gpus"]) == (1, 3, 1)
    assert d["config"]["workload"].startswith("ternary_4b: 2560->9728, 9728->2560 x M in [8192, 1024, 128, 16, 1]")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, ["--gpus", "2"])
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_profiled_traffic_needs_the_captured_source(tmp_path, monkeypatch):
    # The roofline's DRAM traffic comes from a committed machine-readable ncu
    # summary and is reported only while the kernel source still has the hash
    # recorded there.
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src_dir = tmp_path / "binary_weight_transformer_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = src_dir / "kernel.cu"
    src.write_bytes(b"// kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "roofline_traffic.json").write_text(json.dumps(
        {"k M=1": {"source": "kernel.cu", "source_sha256_16": sha, "traffic_bytes_per_launch": 140271360}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k M=1") == 140271360
    assert bench.profiled_traffic("k M=2") is None
    src.write_bytes(b"// kernel v2\n")
    assert bench.profiled_traffic("k M=1") is None


def test_committed_roofline_profiles_match_their_sources():
    # Every entry the bench's roofline can use must describe a committed
    # kernel source and name the summary and the command it came from.
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
        entries = json.load(f)
    assert entries
    for key, e in entries.items():
        assert bench.profiled_traffic(key) == e["traffic_bytes_per_launch"] > 0, key
        assert os.path.exists(os.path.join(ROOT, "profiles", e["summary"])), key
        assert e["command"].startswith("ncu ") and "--clock-control none" in e["command"], key


def test_gpus_flag_launches_that_many_ranks():
    # --gpus 2 without a torchrun environment relaunches the script under
    # torch.distributed.run with two ranks; rank 0 alone prints the line.
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_gpus_flag_must_match_the_launch():
    r = _run({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"}, ["--gpus", "4"])
    assert r.returncode != 0
