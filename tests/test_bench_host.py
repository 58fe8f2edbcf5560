"""Host-side logic of bench.py on CPU: the multi-rank reductions (world size
2 over gloo), the byte model, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    w, r, _ = bench.dist_env()
    bench.barrier(w)
    mx = bench.max_over_ranks(10.0 + r, w)
    sm = bench.sum_over_ranks(1.5 * (r + 1), w)
    with open(f"{out_path}.{r}", "w") as f:
        json.dump({"max": mx, "sum": sm, "world": w}, f)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_reductions(tmp_path):
    port = _free_port()
    out = str(tmp_path / "res")
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    for r in range(2):
        d = json.load(open(f"{out}.{r}"))
        assert d == {"max": 11.0, "sum": 4.5, "world": 2}


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.sum_over_ranks(3.25, 1) == 3.25


def test_byte_model():
    # DeepSeek-V3 shape: 528.5 MB each way
    assert bench.dispatch_bytes(4096, 7168, 8, 32768, False) == 528482304
    assert bench.combine_bytes(4096, 7168, 8) == 528482304
    assert bench.row_bytes(7168, True) == 7168 + 56 * 4


def test_reference_arm_line():
    env = dict(os.environ)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3",
                        "--config", "tiny"], cwd=ROOT, capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0


def test_reference_arm_other_ranks_are_silent():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "3", "--config", "tiny"], cwd=ROOT, capture_output=True, text=True,
                       env=env, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_floor():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_clock_sampler_with_fake_nvml(monkeypatch):
    """Clock sampling reads NVML only (a fake here): a sample on entry and on
    exit even for a short region, event-reason bits mapped to names, the
    interpreter's switch interval restored."""
    import sys
    import time
    import types

    import bench

    unexpected = []

    class FakeNvml(types.ModuleType):
        NVML_CLOCK_SM = 0

        def nvmlInit(self):
            pass

        def nvmlDeviceGetHandleByIndex(self, i):
            return ("dev", i)

        def nvmlDeviceGetMaxClockInfo(self, h, kind):
            return 1965

        def nvmlDeviceGetClockInfo(self, h, kind):
            return 1950

        def nvmlDeviceGetCurrentClocksEventReasons(self, h):
            return 0x4 | 0x1                     # sw_power_cap + idle

        def __getattr__(self, name):             # anything else (a setter, a reset) is recorded
            unexpected.append(name)
            raise AttributeError(name)

    fake = FakeNvml("pynvml")
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    before = sys.getswitchinterval()
    s = bench.ClockSampler(0)
    with s:
        time.sleep(0.01)
    out = s.summary()
    assert out["samples"] >= 2 and out["sm_mhz"] == 1950 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert sys.getswitchinterval() == before
    assert unexpected == []                      # read-only: no other NVML call


def test_kernel_figures_writeback_arithmetic():
    """with_writeback charges each kernel (flush right after it) - (flush of a
    clean L2); fractions divide algorithmic bytes by time and the peak."""
    import bench
    import workloads
    wl = workloads.generate("dsv3", with_x=False)
    ms = lambda v: [v * 1e-3] * 3  # noqa: E731  (µs -> ms samples)
    split = {"layout": ms(13.0), "dispatch": ms(90.0), "combine": ms(80.0),
             "flush_after_dispatch": ms(50.0), "flush_after_combine": ms(42.0), "flush_clean": ms(40.0),
             "dispatch_reuse": ms(88.0)}
    f = bench.kernel_figures(wl, 32768, split, False, 6500.0)
    b = 528482304
    assert f["bytes_per_call"] == {"dispatch": b, "combine": b}
    assert f["us_per_call"] == {"layout": 13.0, "dispatch": 90.0, "combine": 80.0, "dispatch_on_reused_layout": 88.0}
    wb = f["with_writeback"]
    assert wb["dispatch_us"] == 100.0 and wb["combine_us"] == 82.0
    assert abs(wb["dispatch_gbs"] - b / 100e-6 / 1e9) < 0.1
    assert abs(wb["dispatch_frac"] - b / 100e-6 / 1e9 / 6500.0) < 1e-4
    assert abs(f["frac_of_8tbs"]["combine"] - b / 80e-6 / 1e9 / 8000.0) < 1e-4
    # a flush that ran faster than the clean one charges nothing
    split["flush_after_combine"] = ms(39.0)
    assert bench.kernel_figures(wl, 32768, split, True, 6500.0)["with_writeback"]["combine_us"] == 80.0


def test_kernel_digest_ignores_comments_only(tmp_path, monkeypatch):
    """The digest that stamps the recorded DRAM traffic changes with the step
    kernels' code, not with their comments."""
    import shutil
    csrc = tmp_path / "combine_ep_get_08_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.STEP_KERNEL_SOURCES:
        shutil.copy(os.path.join(ROOT, "combine_ep_get_08_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.kernel_source_digest()
    f = csrc / "combine.cu"
    text = f.read_text()
    f.write_text("// a new comment line\n" + text.replace("namespace ep {", "namespace ep {  /* note */", 1) + "\n\n")
    assert bench.kernel_source_digest() == d0
    f.write_text(text.replace("kLoadsInFlight = 8", "kLoadsInFlight = 4", 1))
    assert bench.kernel_source_digest() != d0


def test_expert_gemm_summary_arithmetic(monkeypatch, tmp_path):
    """TFLOP/s of the expert GEMM entries: 2 x (non-masked pairs) x N x I per
    call over the mean event time; the E4M3 peak is twice the measured bf16
    burst (the nominal dense FP8 / bf16 ratio)."""
    import types

    import numpy as np
    import torch
    peaks = tmp_path / "MEASURED_PEAKS.json"
    peaks.write_text(json.dumps({"bf16_tflops": 1600.0, "hbm_gbs": 6500.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.gemm_peak(False)[0] == 1600.0 and bench.gemm_peak(True)[0] == 3200.0
    idx = torch.from_numpy(np.array([[0, 1], [2, -1]], np.int64))    # 3 real pairs
    wl = types.SimpleNamespace(topk_idx=idx)
    for fp8, peak in ((False, 1600.0), (True, 3200.0)):
        o = {"wl": wl, "N": 1024, "I": 512, "fp8": fp8}
        e = bench.expert_gemm_summary(o, [0.002, 0.004])                # mean 3 us
        want = 2.0 * 3 * 1024 * 512 / 3e-6 / 1e12
        assert abs(e["tflops"] - round(want, 1)) < 1e-9
        assert e["peak"] == peak and abs(e["frac"] - round(want / peak, 4)) < 1e-12
        assert e["dtype"] == ("e4m3" if fp8 else "bf16") and e["us_per_call"] == 3.0
    monkeypatch.setattr(bench, "ROOT", str(tmp_path / "none"))
    assert bench.gemm_peak(False)[0] == 1590.0                         # the fallback without the file
