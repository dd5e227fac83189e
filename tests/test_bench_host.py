"""Host-side parts of bench.py: roofline numerators from the storage formats, the oracle reference arm, the
JSON line."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import pytest  # noqa: E402

import bench  # noqa: E402
from gen import CONFIGS  # noqa: E402


def _rec(out_rows, inp, bits):
    # row record: codes, then inp/64 fp16 scales and inp/64 fp16 biases (16-byte padding is 0 at these sizes)
    return out_rows * (inp * bits // 8 + 4 * (inp // 64))


def test_decode_bytes_per_token_layer_35b():
    H, I, E, K, r, P = 2048, 512, 256, 4, 16, 256
    expert = _rec(2 * I, H, 4) + _rec(H, I, 4)
    assert expert == 1_769_472
    shared_lora = 2 * (r * H * 2 + I * r * 2) + (r * I * 2 + H * r * 2)
    router = _rec(E, H, 8)
    shared_gate = _rec(1, H, 8)
    prerouter = P * H * 2 + P * K * 2 + P * 2 + E * P * 2 + E * 2  # W1 token part, K multi-hot columns, b1, W2, b2
    want = K * expert + expert + shared_lora + router + shared_gate + prerouter
    assert want == 10_835_072
    assert bench.token_layer_bytes(CONFIGS[1]) == want


def test_decode_bytes_per_token_layer_8b():
    H, I, E, K, r, P = 2048, 512, 128, 8, 16, 256
    expert = _rec(2 * I, H, 4) + _rec(H, I, 4)
    want = (K + 1) * expert + 2 * (r * H * 2 + I * r * 2) + (r * I * 2 + H * r * 2) + _rec(E, H, 8) + _rec(1, H, 8) \
        + P * H * 2 + P * K * 2 + P * 2 + E * P * 2 + E * 2
    assert want == 17_570_688
    assert bench.token_layer_bytes(CONFIGS[2]) == want


def test_prefill_expert_flops_per_layer():
    T, K, H, I = 3328, 4, 2048, 512
    routed = T * K * (2 * (2 * I) * H + 2 * H * I)
    shared = T * (2 * (2 * I) * H + 2 * H * I)
    assert bench.expert_flops(CONFIGS[3], T) == routed + shared == 104_689_827_840


def _small_decode_cfg():
    import dataclasses

    return dataclasses.replace(CONFIGS[0], T=1, layers=3, lora_routed_down=True)


def test_oracle_work_items_reproduce_the_oracle_stack_pass():
    """The reference arm's item-by-item pass is the oracle's own stack pass, bit for bit."""
    import numpy as np

    from gen import inputs
    from oracle import moe_oracle as O

    cfg = _small_decode_cfg()
    ref = bench.OracleTokenPass(cfg)
    kinds = [ref.step()[0] for _ in range(2 * cfg.layers * (cfg.K + 3))]
    assert kinds[:cfg.K + 3] == ["route"] + ["expert"] * cfg.K + ["shared", "tail"]
    assert len(ref.finished) == 2 and ref.token == 2 and ref.layer == 0 and ref.i == 0
    layers = [inputs.layer(cfg, l) for l in range(cfg.layers)]
    for tok in range(2):
        x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=tok, T=1)).astype(np.float64)
        want = O.stack_forward(x0, layers, cfg.K, eps=bench.EPS)["x"]
        assert np.array_equal(ref.finished[tok], want)


def test_oracle_token_seconds_weights_each_kind_by_its_count():
    cfg = _small_decode_cfg()  # K = 2: a layer is route + 2 experts + shared + tail
    items = [("route", 1.0), ("expert", 2.0), ("expert", 4.0), ("shared", 3.0), ("tail", 0.5), ("route", 3.0)]
    assert bench.oracle_token_seconds(items, cfg) == cfg.layers * (2.0 + 2 * 3.0 + 3.0 + 0.5)
    part = [("route", 1.0), ("expert", 3.0)]  # not every kind sampled: plain item rate
    assert bench.oracle_token_seconds(part, cfg) == 4.0 * cfg.layers * (cfg.K + 3) / 2


def test_reference_arm_prints_one_line_in_the_native_arms_terms(capsys):
    import json

    class Args:
        steps, warmup = 8, 1

    bench.run_reference(Args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "tok/s"
    assert line["steps"] == 8 and line["higher_is_better"] is True and line["value"] > 0
    assert line["e2e"] == {"value": line["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    native = bench.decode_config(CONFIGS[bench.CFG_ID], 1)
    assert {k: line["config"][k] for k in native} == native


def test_cpu_baseline_runs_whole_layers():
    cb = bench.cpu_baseline(CONFIGS[bench.CFG_ID], budget_s=0.0, one_thread_budget_s=1e-9)  # one layer each
    assert cb["kind"] == "oracle" and cb["unit"] == "tok/s" and cb["value"] > 0 and cb["cores"] >= 1
    assert cb["sample"].startswith("1 layer passes")
    assert cb["one_thread"]["cores"] == 1 and cb["one_thread"]["value"] > 0
    assert cb["one_thread"]["sample"].startswith("1 layer passes")
    assert bench.blas_threads() == cb["cores"]  # the limit is lifted again afterwards


def test_clock_sampler_names_the_visible_gpu(monkeypatch):
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    assert bench.smi_gpu_id(3) == "3"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "4,6")
    assert bench.smi_gpu_id(0) == "4" and bench.smi_gpu_id(1) == "6"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-0a1b, GPU-2c3d")
    assert bench.smi_gpu_id(1) == "GPU-2c3d"


def test_clock_sampler_reads_nvml_in_a_thread(monkeypatch):
    """Read-only NVML queries (a fake here) every few ms plus one at each window edge: a window as short as
    a 20-step run still has samples, and the throttle-reason bits map to their names."""
    import sys
    import time
    import types

    import torch

    class FakeNvml(types.ModuleType):
        NVML_CLOCK_SM = 1

        def nvmlInit(self):
            pass

        def nvmlDeviceGetHandleByUUID(self, u):
            assert u == "GPU-1234"
            return "handle"

        def nvmlDeviceGetMaxClockInfo(self, h, c):
            return 1965

        def nvmlDeviceGetClockInfo(self, h, c):
            return 1800

        def nvmlDeviceGetCurrentClocksEventReasons(self, h):
            return 0x4 | 0x1  # sw power cap, and an idle bit that is not a slowdown

    monkeypatch.setitem(sys.modules, "pynvml", FakeNvml("pynvml"))
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: types.SimpleNamespace(uuid="1234"))
    clk = bench.Clocks(torch.device("cpu")).start()
    t0 = time.time()
    clk.edge()
    time.sleep(0.002)
    clk.edge()
    t1 = time.time()
    clk.stop()
    s = clk.summary((t0, t1))
    assert s["samples"] >= 2 and s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["source"] == "nvml"


def test_headline_line_carries_every_contract_key():
    cfg = CONFIGS[bench.CFG_ID]
    steps, ms, world = 2000, 1900.0, 2
    value = bench.whole_job_rate(cfg.T * steps, world, ms)
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    line = bench.headline_line(cfg, world, steps, 20, ms, value, 900.0, True, clocks)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["value"] == pytest.approx(2 * steps / 1.9) and line["ms_per_step"] == pytest.approx(0.95)
    assert line["n_gpus"] == 2 and line["scaling"] == "weak" and line["config"]["parallelism"] == "replicas x2"
    assert line["config"]["workload"] and line["clocks"] is clocks
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["algorithmic_bytes_per_step"] == 433_402_880
    assert r["achieved"] == pytest.approx(433_402_880 / 0.95e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert line["e2e"] == {"value": 900.0, "unit": "tok/s", "h2d_bytes_per_step": 2048 * 4,
                           "d2h_bytes_per_step": 2048 * 4}
    assert line["gpu_launches"] == steps  # one cooperative launch per token
    per_layer = bench.headline_line(cfg, 1, steps, 20, ms, value, 900.0, False, clocks)
    assert per_layer["gpu_launches"] == steps * cfg.layers * 10 and per_layer["roofline"]["traffic"] is None
