"""bench.py's contract pieces that run without a GPU: the reference arm (the
oracle on the host cores) prints its one JSON line, a second rank of it exits
without work, and the algorithmic bytes of the decode stack match the closed
forms of the workload."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _run(extra_env, *args):
    env = dict(os.environ, **extra_env)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=300, cwd=ROOT)


def test_reference_arm_prints_one_json_line():
    r = _run({}, "--impl", "reference", "--layers", "1", "--steps", "2", "--warmup", "0")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["metric"] == bench.METRIC and d["value"] > 0 and 1 <= d["steps"] <= 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and "7 GEMVs" in d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--impl", "reference",
             "--layers", "1", "--steps", "1")
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_stack_algorithmic_bytes_closed_forms():
    codes, total = bench.algorithmic_bytes(bench.stack_spec(16))
    # 973,078,528 weights at 5 bits per 4 weights
    assert codes == 973078528 * 5 // 32 == 152043520
    # + fp32 scales (4 B per row), int8 x (K per GEMV) and fp32 y (4 B per row)
    rows = 16 * (2048 + 512 + 512 + 2048 + 8192 + 8192 + 2048)
    ks = 16 * (6 * 2048 + 8192)
    assert total == codes + 4 * rows + ks + 4 * rows == 155385856


def _sample(uuid, bus, mhz, power_cap="Not Active"):
    return (1.0, uuid, bus, [str(mhz), "1965", "700", "0x0", "Not Active", "Not Active",
                             "Not Active", power_cap])


def test_clock_sampler_matches_the_gpu_by_uuid_or_pci_bus():
    rows = [_sample("GPU-AbCd-0001", "00000000:1B:00.0", 1965),
            _sample("GPU-ffff-0002", "00000009:2C:00.0", 1200, "Active")]
    # torch prints the UUID without the prefix and in lower case
    by_uuid = bench.ClockSampler("abcd-0001", None)
    by_uuid.samples, by_uuid.seen = rows, {r[1]: r[2] for r in rows}
    s = by_uuid.summary(0.0, 2.0)
    assert s["samples"] == 1 and s["sm_mhz"] == 1965.0 and s["reasons"] == []
    # no usable UUID: the PCI domain, bus and device decide
    by_pci = bench.ClockSampler(None, (9, 0x2C, 0))
    by_pci.samples, by_pci.seen = rows, {r[1]: r[2] for r in rows}
    s = by_pci.summary(0.0, 2.0)
    assert s["samples"] == 1 and s["sm_mhz"] == 1200.0 and s["reasons"] == ["sw_power_cap"]
    # nothing matches among several GPUs: no samples rather than another GPU's
    none = bench.ClockSampler("0000", (1, 2, 3))
    none.samples, none.seen = rows, {r[1]: r[2] for r in rows}
    assert none.summary(0.0, 2.0)["samples"] == 0
    # a listing of one GPU is that GPU
    one = bench.ClockSampler("0000", None)
    one.samples, one.seen = rows[:1], {rows[0][1]: rows[0][2]}
    assert one.summary(0.0, 2.0)["samples"] == 1


def test_layer_activations_share_as_a_llama_layer():
    import torch
    spec = [("q", 8, 32), ("k", 4, 32), ("v", 4, 32), ("o", 8, 32), ("gate", 16, 32), ("up", 16, 32),
            ("down", 8, 64)]
    entries = [(l, name, k) for l in range(2) for name, _, k in spec]
    calls = []

    def make(shape, gen):
        calls.append(shape)
        return torch.randint(-127, 128, shape, dtype=torch.int8, generator=gen)

    xs = bench.layer_activations(torch, torch.device("cpu"), entries, 3, make, 5)
    assert len(xs) == 14 and len(calls) == 8          # 4 distinct inputs per layer
    for base in (0, 7):
        q, k, v, o, gate, up, down = xs[base:base + 7]
        assert q is k and k is v and gate is up
        assert len({id(q), id(o), id(gate), id(down)}) == 4
        assert tuple(q.shape) == (3, 32) and tuple(down.shape) == (3, 64)
    assert xs[0] is not xs[7]                          # layers do not share inputs
