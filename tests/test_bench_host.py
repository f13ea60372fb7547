"""CPU checks of bench.py's host logic: the FLOP count behind `value`, the
kernel-source hash that keys the committed DRAM-traffic figures, and the
reference arm's JSON line (the oracle timed on the host cores)."""
import json
import os
import shutil
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_linear_flops_is_the_sum_of_the_layer_products():
    """4MNK + 6Mr(N+K) is every product of one forward and backward, each
    counted as 2 m n k: forward X W'^T, X A, (X A) B; backward dY W' (dX),
    dY B^T, G A^T (the low-rank part of dX), X^T G (dA), (X A)^T dY (dB)."""
    for M, N, K, r in ((2048, 4096, 4096, 64), (16, 11008, 4096, 8), (3, 64, 192, 16)):
        products = [(M, N, K), (M, r, K), (M, N, r),
                    (M, K, N), (M, r, N), (M, K, r), (K, r, M), (r, N, M)]
        assert bench.linear_flops(M, N, K, r) == sum(2 * m * n * k for m, n, k in products)


def _sources():
    return {rel: open(os.path.join(ROOT, rel), encoding="utf-8").read() for rel in bench.KERNEL_SOURCES}


def test_kernel_hash_ignores_comments_and_spacing_only():
    src = _sources()
    base = bench.kernel_source_hash(read=lambda rel: src[rel])
    assert base == bench.kernel_source_hash()
    first = bench.KERNEL_SOURCES[0]
    commented = dict(src)
    commented[first] = "// a new comment line\n" + src[first].replace("\n", "\n  ", 3) + "\n/* block */\n"
    assert bench.kernel_source_hash(read=lambda rel: commented[rel]) == base
    edited = dict(src)
    edited[first] = src[first] + "\nstatic int qlora_hash_probe = 1;\n"
    assert bench.kernel_source_hash(read=lambda rel: edited[rel]) != base


def test_profiled_traffic_only_for_the_profiled_kernels(tmp_path, monkeypatch):
    """The committed traffic figure is reported only while the kernel
    sources still hash to the value it was captured with."""
    for rel in bench.KERNEL_SOURCES:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    (tmp_path / "profiles" / "traffic.txt").write_text(
        f"# summary\nkernel_source_hash: {h}\nqgemm_fwd_gemm: 38810000\nqgemm_bwd_gemm: 41670000\n")
    assert bench.profiled_traffic("qgemm_fwd_gemm") == 38810000.0
    assert bench.profiled_traffic("qgemm_bwd_gemm") == 41670000.0
    assert bench.profiled_traffic("qgemm_other") is None
    with open(tmp_path / bench.KERNEL_SOURCES[0], "a") as f:
        f.write("\nstatic int changed_kernel = 2;\n")
    assert bench.profiled_traffic("qgemm_fwd_gemm") is None


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_json_line():
    p = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["n_gpus"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == bench.WORKLOAD
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    """Under torchrun only rank 0 runs and prints the reference arm."""
    p = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "0", "--gpus", "2"],
                   {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
