"""The benchmark's JSON line (host side): the reference arm, which times the
CPU oracle, prints one line with the keys the benchmark contract fixes."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "resnet18_layer2_3x3_c128_n64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_algorithmic_bytes_and_flops_of_the_benchmark_layer():
    """The roofline's numerators for the 28x28, 128->128, N = 64, 3x3 NVFP4
    layer, by hand: X and G_Y 28·28·128·64 = 6,422,528 elements, W
    128·9·128 = 147,456; quantize 8.5625 B per element (two fp32 reads, a
    half-byte code, 1/16 of a scale byte); each conv pass reads both
    quantized operands once (0.5625 B per element) and writes its fp32
    output once; 2·128·128·9·28·28·64 FLOPs per pass."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    layer = workloads.resnet18_layer2()
    quant, conv, (x, w, g) = bench.layer_bytes(layer)
    assert (x, w, g) == (6422528, 147456, 6422528)
    assert sum(quant.values()) == 12992512 * 8.5625 == 111248384
    assert conv == {"fwd": 6569984 * 0.5625 + 6422528 * 4,
                    "wgrad": 12845056 * 0.5625 + 147456 * 4,
                    "dgrad": 6569984 * 0.5625 + 6422528 * 4}
    assert conv["fwd"] == 29385728 and conv["wgrad"] == 7815168
    assert layer.flops() == 2 * 128 * 128 * 9 * 28 * 28 * 64 == 14797504512
