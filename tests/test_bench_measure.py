"""bench.py's measure() arithmetic on one process, with the device pieces
stood in: value = outputs / device time per step, e2e from its own time,
launch count = launches per step x steps, traffic from the committed record."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_measure_single_process(monkeypatch):
    spec = importlib.util.spec_from_file_location("bench_measure", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)

    class Wl:
        name, B, H, N, dtype, gated, D = "w", 1, 4, 1024, "f32", False, None

        def io_bytes(self):
            return 8 * 4096

    class Runner:
        outputs = 4096

        class plan:
            path, mma_flops = "fused", 1.0e9

        def __init__(self, *a, **k):
            pass

        def step(self, **k):
            pass

        def dominant_kernel(self):
            return "fused_fwd_simt"

        def compute_dtype(self):
            return "f32"

        def launches_per_step(self):
            return 2

    class Cuda:
        @staticmethod
        def synchronize():
            pass

        @staticmethod
        def empty_cache():
            pass

    class Torch:
        cuda = Cuda
        float32 = None

        @staticmethod
        def empty(*a, **k):
            return None

    class Args:
        kernel, shard = "auto", "weak"

    monkeypatch.setattr(b, "Runner", Runner)
    monkeypatch.setattr(b, "time_steps", lambda r, steps, torch, flush: [0.002] * steps)
    monkeypatch.setattr(b, "time_e2e", lambda r, steps, torch: (0.01, 16384, 16384))
    monkeypatch.setattr(b, "workload_config", lambda wl, path, world, shard: {"workload": wl.name})
    res = b.measure(Wl(), Args, Torch, 5, 3, pg=None, world=1, clocks=False, e2e=True, cpu_seconds=0.0,
                    config_name="pr1_b1_h4_n1024_f32")
    assert abs(res["value"] - 4096 / 2e-6) < 1e-3
    assert abs(res["ms_per_step"] - 0.002) < 1e-12
    assert abs(res["e2e"]["value"] - 4096 / 1e-5) < 1e-3 and res["e2e"]["h2d_bytes_per_step"] == 16384
    assert res["gpu_launches"] == 10
    roof = res["roofline"]
    assert roof["bound"] == "hbm" and abs(roof["achieved"] - round(8 * 4096 / 2e-6 / 1e9, 1)) < 1e-9
    assert roof["traffic"] == b.recorded_traffic("pr1_b1_h4_n1024_f32", "fused_fwd_simt")
    assert abs(res["tensor_pipe"]["achieved_tflops"] - round(1.0e9 / 2e-6 / 1e12, 2)) < 1e-9
