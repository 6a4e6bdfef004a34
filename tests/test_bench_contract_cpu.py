"""bench.py's reference arm (the fp64 oracle on the host cores) prints one JSON line with the
fields the benchmark contract names; the own arm needs a GPU and is exercised by the GPU runs."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "tiny" in d["config"]["workload"]


def _bench_module():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_source_hash_ignores_comments_and_blank_lines(tmp_path, monkeypatch):
    """The roofline's `traffic` stays valid across comment edits and goes null on a code edit."""
    import shutil
    bench = _bench_module()
    src = os.path.join(ROOT, "mixture_experts_routed_04_b200", "csrc")
    dst = tmp_path / "mixture_experts_routed_04_b200" / "csrc"
    shutil.copytree(src, dst, ignore=shutil.ignore_patterns("*.o", "*.so"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = bench.kernel_source_hash(bench.STREAM_SRC)
    f = dst / "stream.cu"
    text = f.read_text()
    f.write_text("// a comment line\n\n" + text.replace("\n", "  // trailing note\n", 1))
    assert bench.kernel_source_hash(bench.STREAM_SRC) == before
    f.write_text(text + "\nstatic int an_added_line = 0;\n")
    assert bench.kernel_source_hash(bench.STREAM_SRC) != before


def test_committed_traffic_reads_the_rows_of_the_current_sources():
    """Every row of the DRAM-traffic table taken on the current kernel source is what bench.py
    reports as `traffic` (read + write bytes per launch); rows of other sources are not used."""
    bench = _bench_module()
    sources = {"tc_gateup": bench.ONE_SM_SRC, "tc_down": bench.ONE_SM_SRC,
               "stream_gateup": bench.STREAM_SRC, "stream_down": bench.STREAM_SRC}
    with open(os.path.join(ROOT, "profiles", "dram_traffic.md")) as fh:
        for line in fh:
            cells = [c.strip().strip("`") for c in line.strip().strip("|").split("|")]
            if len(cells) < 5 or cells[0] not in sources or not cells[3].isdigit():
                continue
            kern, cfg, h, rd, wr = cells[:5]
            if h == bench.kernel_source_hash(sources[kern]):
                assert bench.committed_traffic(kern, sources[kern], cfg) == int(rd) + int(wr)
    # a workload without a row gives no traffic
    assert bench.committed_traffic("tc_gateup", bench.ONE_SM_SRC, "no_such_workload") is None
