"""Host logic of bench.py (no GPU): the algorithmic byte model, the source hash
that ties a profile to the kernel it measured, the clock / power parsing, the
time-bounded oracle timing and the reference arm's JSON line."""
import importlib.util
import json
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _flat(optimizer, ecc_bits, n):
    from workloads.shapes import ADAMW_HP, SGDM_HP, TensorSpec, Workload

    hp = dict(ADAMW_HP) if optimizer == "adamw" else dict(SGDM_HP)
    return Workload(name="flat", tensors=[TensorSpec("t", (n,), "normal", 0.02)], optimizer=optimizer,
                    hparams=hp, ecc_bits=ecc_bits)


@pytest.mark.parametrize("opt,nbits,per_param", [("adamw", 8, 12.25), ("adamw", 16, 14.25), ("sgdm", 8, 10.125)])
def test_algorithmic_bytes_per_parameter(bench, opt, nbits, per_param):
    # whole groups: the per-parameter figures of the traffic model (FlashOptim
    # blog, "Methodology": 16-bit downcast + 8/16-bit ECC, 8-bit states with one
    # 16-bit scale per 32 elements, gradients read in backward precision)
    n = 32 * 1000
    assert bench.algorithmic_bytes(_flat(opt, nbits, n)) == per_param * n
    # a partial last group still carries a whole scale per state
    one = {"adamw": {8: 12 + 8, 16: 14 + 8}, "sgdm": {8: 10 + 4}}[opt][nbits]
    assert bench.algorithmic_bytes(_flat(opt, nbits, 1)) == one
    assert bench.algorithmic_bytes(_flat(opt, nbits, n + 1)) == per_param * n + one


def test_default_workload_bytes(bench):
    from workloads import workload

    wl = workload("llama3.1-8b")
    assert wl.numel == 8_030_261_248
    assert bench.algorithmic_bytes(wl) == 98_370_700_288


def _copy_sources(tmp_path):
    root = tmp_path / "r"
    (root / "bit_states_b200" / "csrc").mkdir(parents=True)
    (root / "profiles").mkdir()
    for f in ("fo_codec.cuh", "fo_kernels.cuh", "fo_api.cu"):
        shutil.copy(os.path.join(ROOT, "bit_states_b200", "csrc", f), root / "bit_states_b200" / "csrc" / f)
    return root


def test_source_sha_ignores_comments_only(bench, tmp_path, monkeypatch):
    root = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    base = bench.kernel_source_sha()
    k = root / "bit_states_b200" / "csrc" / "fo_kernels.cuh"
    src = k.read_text()
    k.write_text(src + "\n// a comment\n/* and\n another */\n")
    assert bench.kernel_source_sha() == base
    k.write_text(src + "\nconstexpr int fo_sha_probe = 1;\n")
    assert bench.kernel_source_sha() != base


def test_traffic_attached_only_to_the_measured_source(bench, tmp_path, monkeypatch):
    root = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_sha()
    prof = {"cfg": {"kernel_source_sha": sha, "dram_bytes_per_launch": 1234}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(prof))
    assert bench.traffic_from_profile("cfg") == 1234
    assert bench.traffic_from_profile("other") is None
    prof["cfg"]["kernel_source_sha"] = "0" * 16
    (root / "profiles" / "traffic.json").write_text(json.dumps(prof))
    assert bench.traffic_from_profile("cfg") is None


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_sampler_parsing(bench, tmp_path):
    rows = []
    # idle, a ramp, then a steady plateau at the power limit with the cap reason active
    for sm, pw in [(1965, 150.0), (1965, 400.0), (1900, 800.0), (1700, 990.0), (1690, 1000.0), (1680, 1001.0),
                   (1675, 999.0)]:
        cap = "Active" if pw > 900 else "Not Active"
        rows.append(f"0, {sm}, 1965, {pw}, 0x4, Not Active, Not Active, Not Active, {cap}")
    path = tmp_path / "clk.csv"
    path.write_text("\n".join(rows) + "\n")
    s = bench.ClockSampler("0")
    s.proc = _DoneProc()
    s.path = str(path)
    c = s.stop()
    assert c["samples"] == 7
    assert c["samples_under_load"] == 6           # above 200 W
    assert c["sm_mhz"] == 1695.0                  # median of the loaded samples
    assert c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert c["power_w_max"] == 1001.0
    assert c["power_w_steady"] == 1000.0          # second half of the loaded samples
    assert c["power_w_median"] == 994.5
    assert not path.exists()


def test_time_oracle_runs_until_the_time_bound(bench):
    wl = _flat("adamw", 8, 1 << 16)
    value, dt, n, k = bench.time_oracle(wl, 1 << 14, 1, 1, 2, min_seconds=0.3)
    assert dt >= 0.3 and k >= 2 and n == 1 << 14
    assert value == pytest.approx(n * k / dt / 1e9)


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "1", "--config", "flat-1M", "--cpu-sample-params", "65536"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "Gparams/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "Gparams/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("flat-1M")
