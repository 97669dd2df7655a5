"""bench.py's reference arm (the oracle timed on the host cores) and its
host-side helpers, on the CPU: the printed line carries the contract's keys,
non-zero ranks print nothing, and the FLOP / byte model matches closed forms."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *args):
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]


def test_reference_line_keys_tiny_workload():
    lines = _run({}, "--workload", "tiny_h2_n1024", "--steps", "1", "--warmup", "0")
    assert len(lines) == 1
    ln = lines[0]
    assert ln["impl"] == "reference" and ln["unit"] == "TFLOPS" and ln["higher_is_better"] is True
    assert ln["value"] > 0 and ln["ms_per_step"] > 0 and ln["steps"] == 1
    assert ln["config"]["workload"] == "tiny_h2_n1024"
    cb = ln["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == ln["value"] and cb["cores"] >= 1 and cb["sample"]
    assert cb["extrapolated"] is True and ln["ms_per_step_extrapolated"] is True
    e2e = ln["e2e"]
    assert e2e["value"] == ln["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_loads_only_the_oracle_library():
    """The reference arm maps the oracle's library and never the product's."""
    code = (f"import sys, runpy; sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'tiny_h2_n1024', "
            f"'--steps', '1', '--warmup', '0']; sys.path.insert(0, {ROOT!r}); "
            f"\ntry:\n    runpy.run_path({os.path.join(ROOT, 'bench.py')!r}, run_name='__main__')\n"
            f"except SystemExit:\n    pass\n"
            f"maps = open('/proc/self/maps').read(); print('LIBS', 'liboracle.so' in maps, 'libsagesla.so' in maps)")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert "LIBS True False" in r.stdout, r.stdout[-1000:] + r.stderr[-2000:]


def test_reference_arm_other_ranks_print_nothing():
    assert _run({"RANK": "1"}, "--workload", "tiny_h2_n1024", "--steps", "1", "--warmup", "0") == []


def test_flop_and_byte_model_closed_forms():
    sys.path.insert(0, ROOT)
    import bench
    from oracle import oracle as orc
    w = bench.workloads()["wan2.1-14b-720p_h40_n75600"]
    f = bench.flops(w, orc.topk_count(1182, w.topk))
    BH, N, d = 40, 75600, 128
    nb = (N + 63) // 64
    assert f["nb"] == nb == 1182 and f["kc"] == 119
    assert f["dense"] == 4.0 * BH * N * N * d
    assert f["computed"] == 4.0 * BH * nb * 119 * 64 * 64 * d
    E = BH * N * d
    assert f["hbm_bytes"] == 18.0 * E
