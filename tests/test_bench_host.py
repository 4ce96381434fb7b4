"""Host logic of the benchmark.

- Whether a committed ncu figure still describes the kernels: the code
  digest ignores comments and whitespace, follows any change of code, and
  the recorded DRAM traffic is read only while the digest matches.
- The reference arm (the fp64 oracle on the host cores): its JSON line,
  the same config object as the device arm, and that only rank 0 prints it.
- --gpus N must match the launcher's world size."""
import os

import bench


def test_code_tokens_drop_comments_and_whitespace():
    a = "int x = 1;  // one\n/* block\n comment */ float y=2;\n"
    b = "int x = 1;\nfloat y=2; // other words\n"
    assert bench.code_tokens(a) == bench.code_tokens(b)
    assert bench.code_tokens(a) == "int x = 1; float y=2;"


def test_code_change_changes_the_digest():
    files = bench.KERNEL_SOURCES["mid_tc"]
    real = {}
    for f in files:
        with open(os.path.join(bench.ROOT, "nystr_self_attention_segment_b200", "csrc", f)) as fh:
            real[f] = fh.read()
    base = bench.source_digest("mid_tc")
    assert bench.source_digest("mid_tc", real.get) == base
    commented = dict(real)
    commented[files[-1]] = "// a new comment line\n" + real[files[-1]] + "\n/* trailing */\n"
    assert bench.source_digest("mid_tc", commented.get) == base
    edited = dict(real)
    edited[files[-1]] = real[files[-1]].replace("kStages = 6", "kStages = 5", 1)
    assert edited[files[-1]] != real[files[-1]]
    assert bench.source_digest("mid_tc", edited.get) != base


def test_recorded_traffic_needs_a_matching_digest(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "mid_tc_w.md").write_text(
        "traffic_bytes: 1234\nsource_digest: `%s`\n" % bench.source_digest("mid_tc"))
    (prof / "mid_tc_stale.md").write_text("traffic_bytes: 1234\nsource_digest: `0000`\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the digest reads the sources under ROOT too: give it the real tree
    real_root = os.path.dirname(os.path.abspath(bench.__file__))
    os.symlink(os.path.join(real_root, "nystr_self_attention_segment_b200"),
               tmp_path / "nystr_self_attention_segment_b200")
    assert bench.recorded_traffic("mid_tc", "w") == 1234
    assert bench.recorded_traffic("mid_tc", "stale") is None
    assert bench.recorded_traffic("mid_tc", "absent") is None


def _run_bench(args, env_extra=None, rc=0):
    import json
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py")] + args,
                       capture_output=True, text=True, timeout=300, env=env, cwd=bench.ROOT)
    if rc != 0:
        assert r.returncode != 0
        return r.stderr
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    return lines


def test_reference_arm_line_on_the_host():
    # The reference arm times the fp64 oracle on the host cores and prints
    # the contract's line with impl, cpu_baseline and a zero-copy e2e.
    (line,) = _run_bench(["--impl", "reference", "--workload", "tiny_f32_m8",
                          "--steps", "2", "--warmup", "1"])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 2 and line["warmup"] == 1
    assert line["config"]["workload"] == "tiny_f32_m8"
    from nystr_self_attention_segment_b200.inputs import WORKLOADS
    assert line["config"] == bench.workload_config(WORKLOADS["tiny_f32_m8"], 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_prints_on_rank_zero_only():
    assert _run_bench(["--impl", "reference", "--workload", "tiny_f32_m8", "--steps", "1",
                       "--warmup", "0", "--gpus", "2"], {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_gpus_must_match_the_world_size():
    err = _run_bench(["--impl", "reference", "--workload", "tiny_f32_m8", "--steps", "1",
                      "--warmup", "0", "--gpus", "2"], {"RANK": "0", "WORLD_SIZE": "1"}, rc=1)
    assert "WORLD_SIZE" in err
    err = _run_bench(["--impl", "reference", "--workload", "tiny_f32_m8", "--steps", "1",
                      "--warmup", "0"], {"RANK": "0", "WORLD_SIZE": "4"}, rc=1)
    assert "--gpus 1" in err
