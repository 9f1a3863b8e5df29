"""Host-side checks of bench.py that need no GPU: the byte accounting, the
source digest that keys the recorded DRAM traffic, the traffic recorder's
CSV parsing, and the reference arm's JSON line."""
import json
import os
import shutil
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_weight_bytes_of_the_decode_sweep():
    # 0.5 B per weight + one fp16 scale per 128 weights
    assert bench.weight_bytes(4096, 4096) == 8_650_752
    assert bench.weight_bytes(11008, 4096) == 23_248_896
    assert bench.weight_bytes(4096, 11008) == 23_248_896
    assert bench.step_weight_bytes() == 4 * (8_650_752 + 2 * 23_248_896)


def test_code_only_drops_comments_not_strings():
    src = 'int a; // note\n/* block\n comment */ int b;\n\nasm("x // not a comment");\n'
    out = bench._code_only(src)
    assert "note" not in out and "block" not in out
    assert 'asm("x // not a comment");' in out
    assert out.splitlines() == ["int a;", " int b;", 'asm("x // not a comment");']


@pytest.fixture()
def tree(tmp_path, monkeypatch):
    """A copy of the CUDA sources under a temporary root."""
    d = tmp_path / "w4a16_gemm_fp4_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "w4a16_gemm_fp4_b200", "csrc"), d,
                    ignore=shutil.ignore_patterns("*.o", "*.so"))
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_source_digest_ignores_comments_only(tree):
    f = tree / "w4a16_gemm_fp4_b200" / "csrc" / "common.cuh"
    base = bench.kernel_sources_sha()
    f.write_text(f.read_text() + "\n// a remark\n/* and another */\n")
    assert bench.kernel_sources_sha() == base
    f.write_text(f.read_text() + "\nconstexpr int kUnused = 1;\n")
    assert bench.kernel_sources_sha() != base


def _ncu_csv(path, names, values):
    head = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
            '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')
    lines = ["==PROF== Connected to process 1\n", head]
    for i, (name, (rd, wr)) in enumerate(zip(names, values)):
        for metric, v in (("dram__bytes_read.sum", rd), ("dram__bytes_write.sum", wr)):
            lines.append('"%d","1","python","h","void %s(Params)","1","7","(256, 1, 1)","(148, 1, 1)","0",'
                         '"10.0","Command line profiler metrics","%s","byte","%d"\n' % (i, name, metric, v))
    path.write_text("".join(lines))


def test_record_traffic_reads_the_first_sweep(tree, tmp_path):
    from w4a16_gemm_fp4_b200 import api, build
    build.build()
    api.lib()
    keys = [(i, M) for M in bench.MS for i in range(len(bench.SHAPES))]
    bases = [bench.gemm_kernel_name(api, M, *bench.SHAPES[i]).split("<")[0] for (i, M) in keys]
    values = [(1000 + 10 * n, 7 * n) for n in range(len(keys))]
    # one capture per kernel (as traffic_cmds() runs them), its launches in key order
    paths = []
    for base in sorted(set(bases)):
        mine = [n for n in range(len(keys)) if bases[n] == base]
        csv = tmp_path / ("traffic_%s.csv" % base)
        _ncu_csv(csv, [base + "<1, 1>" for _ in mine], [values[n] for n in mine])
        paths.append(str(csv))
    assert len(paths) == len(bench.traffic_cmds())
    bench.record_traffic(",".join(paths))
    doc = json.loads((tree / "profiles" / "traffic.json").read_text())
    assert doc["sources_sha"] == bench.kernel_sources_sha()
    assert len(doc["launches"]) == len(keys)
    for n, (i, M) in enumerate(keys):
        N, K = bench.SHAPES[i]
        e = doc["launches"]["%s %dx%d M=%d" % (bench.gemm_kernel_name(api, M, N, K), N, K, M)]
        assert e["dram_bytes"] == values[n][0] + values[n][1]
        assert e["algorithmic_bytes"] == bench.weight_bytes(N, K) + M * K * 2 + M * N * 2
    # the bench reads the entry back while the sources are unchanged
    k0 = "%s %dx%d M=%d" % (bench.gemm_kernel_name(api, 1, 4096, 4096), 4096, 4096, 1)
    assert bench.recorded_traffic(k0) == values[0][0] + values[0][1]


def test_reference_arm_json_line():
    """`--impl reference` times the oracle on the host and prints the base
    contract's line with impl, cpu_baseline and a zero-copy e2e."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_launches_per_call_counts_the_prepass():
    """The bench's launch count: one kernel per decode-engine call and per
    64-token call, two (f16 pre-pass + GEMM) for the other tensor tiles."""
    from w4a16_gemm_fp4_b200 import api
    calls = {(M, N, K): bench.launches_per_call(api, M, N, K) for M in bench.MS for (N, K) in bench.SHAPES}
    for (M, N, K), n in calls.items():
        decode = api.gemm_engine_for(M, N, K, bench.GROUP) == api.ENGINE_DECODE
        assert n == (1 if decode or 32 < M <= 64 else 2), (M, N, K, n)
    # the sweep: M = 16 on all three matrices takes the tensor engine's 16-token tile
    assert sum(calls.values()) == 15
