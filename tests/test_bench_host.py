"""Host-side checks of bench.py (no GPU): every name it loads is bound, the
roofline arithmetic, and the reference arm (the CPU oracle) end to end."""
import ast
import builtins
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _bound_names(tree):
    names = set(dir(builtins)) | {"__file__", "__name__"}
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            names.add(node.name)
            if not isinstance(node, ast.ClassDef):
                a = node.args
                for arg in a.args + a.kwonlyargs + a.posonlyargs + ([a.vararg] if a.vararg else []) + \
                        ([a.kwarg] if a.kwarg else []):
                    names.add(arg.arg)
        elif isinstance(node, ast.Lambda):
            for arg in node.args.args:
                names.add(arg.arg)
        elif isinstance(node, (ast.Import, ast.ImportFrom)):
            for al in node.names:
                names.add((al.asname or al.name).split(".")[0])
        elif isinstance(node, ast.Name) and isinstance(node.ctx, (ast.Store, ast.Del)):
            names.add(node.id)
        elif isinstance(node, ast.ExceptHandler) and node.name:
            names.add(node.name)
    return names


def test_bench_has_no_unbound_names():
    for f in ("bench.py", "__graft_entry__.py"):
        tree = ast.parse(open(os.path.join(ROOT, f)).read())
        bound = _bound_names(tree)
        unbound = sorted({n.id for n in ast.walk(tree) if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load)
                          and n.id not in bound})
        assert not unbound, f"{f}: {unbound}"


def test_roofline_arithmetic():
    import bench
    from mixture_experts_routed_moe_b200 import inputs as G

    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}
    wl = G.WORKLOADS["decode"]
    r = bench.stage_roofline(wl, "decode", {1: 0.1, 2: 0.05}, 40, peaks, "measured")
    byts = 40 * 2 * wl.I * wl.H * 2 + wl.T * wl.H * 2 + wl.A * wl.I * 2
    assert r["bound"] == "hbm" and r["stage"] == "gate_up"
    assert abs(r["achieved"] - byts / 1e-4 / 1e9) < 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 6000.0) < 1e-12
    wl = G.WORKLOADS["prefill"]
    r = bench.stage_roofline(wl, "prefill", {1: 0.3, 2: 0.2}, 128, peaks, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 4 * wl.A * wl.H * wl.I / 3e-4 / 1e12) < 1e-6 * r["achieved"]
    # the FP8 layer streams more weight bytes than its FLOPs need at the fp8
    # peak: bound by HBM, algorithmic bytes = touched weights + scales + x + h
    wl = G.WORKLOADS["fp8"]
    r = bench.stage_roofline(wl, "prefill", {1: 2.0, 2: 1.0}, 256, peaks, "measured")
    H, I, A = wl.H, wl.I, wl.A
    byts = 256 * 2 * I * H + A * H + A * I + 256 * (2 * I // 128) * (H // 128) + A * (H // 128) * 4 + A * (I // 128) * 4
    assert r["bound"] == "hbm" and r["stage"] == "gate_up" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - byts / 2e-3 / 1e9) < 1e-6 * r["achieved"]
    assert 4 * A * H * I / (3000.0 * 1e12) < byts / (6000.0 * 1e9)
    # e4m3 decode: weight codes plus one scale byte per 128x128 block
    wl = G.WORKLOADS["fp8_decode"]
    r = bench.stage_roofline(wl, "decode", {1: 0.5, 2: 0.25}, 90, peaks, "measured")
    byts = 90 * 2 * wl.I * wl.H + 90 * (2 * wl.I // 128) * (wl.H // 128) + wl.T * wl.H * 2 + wl.A * wl.I
    assert r["kernel"] == "decode_e4m3_gate_up_kernel"
    assert abs(r["achieved"] - byts / 5e-4 / 1e9) < 1e-6 * r["achieved"]
    # the fused path: one kernel streams every touched expert's three matrices
    wl = G.WORKLOADS["decode"]
    r = bench.stage_roofline(wl, "fused", {1: 0.15, 2: 0.0}, 42, peaks, "measured")
    byts = 42 * 3 * wl.I * wl.H * 2 + 2 * wl.T * wl.H * 2
    assert r["kernel"] == "fused_decode_kernel" and r["bound"] == "hbm"
    assert abs(r["achieved"] - byts / 1.5e-4 / 1e9) < 1e-6 * r["achieved"]


def test_reference_arm_runs_on_cpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
