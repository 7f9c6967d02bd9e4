"""Host-side arithmetic of the benchmark (CPU only): the per-kernel algorithmic work that
the roofline fractions divide by, pinned to figures computed independently from the layer
shapes, and the source digest that decides whether the committed ncu traffic still applies."""
import os
import types

import pytest

import bench
from mixture_experts_layer_65_b200 import workloads as W


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _gb(x):
    return x / 1e9


def _shape(name: str):
    """The layer's sizes without drawing its tensors."""
    return types.SimpleNamespace(name=name, **W.CONFIGS[name])


@pytest.mark.parametrize("name,gflop", [
    ("2b", 451.0), ("gshard", 451.0), ("16b_prefill", 2268.0), ("145b", 19791.0)])
def test_expert_gemm_flops_of_the_layers(name, gflop):
    # 6 d I (K_s + K') FLOPs per token: three d x I products per selected expert, 2 FLOPs
    # per multiply-add; 2B and GShard-like layers are iso-compute by construction
    work = bench.algorithmic_work(_shape(name))
    assert work["gate_up_gemm"][0] == "tensor" and work["down_gemm"][0] == "tensor"
    total = work["gate_up_gemm"][1] + work["down_gemm"][1]
    assert abs(total / 1e9 - gflop) / gflop < 1e-3
    assert work["gate_up_gemm"][1] == pytest.approx(2 * work["down_gemm"][1])


def test_memory_bound_bytes_of_the_16b_layer():
    work = bench.algorithmic_work(_shape("16b_prefill"))
    T, d = 16384, 2048
    # router: token matrix + centroids read, (index, gate, rank) per selected slot written
    assert work["router"] == ("hbm", T * d * 2 + 64 * d * 2 + T * 6 * 12)
    assert _gb(work["router"][1]) == pytest.approx(0.0685, abs=5e-4)
    # permute: each token row read once, written once per selected expert
    assert _gb(work["permute"][1]) == pytest.approx(0.470, abs=1e-3)
    # combine: u, the shared output, K' routed rows read, h written, slots and gates read
    assert _gb(work["combine"][1]) == pytest.approx(0.604, abs=1e-3)


def test_decode_sized_gemms_are_counted_as_weight_streams():
    w = _shape("16b_decode")
    work = bench.algorithmic_work(w, active_experts=64)
    # one kernel runs both GEMMs: its slot (gate/up) carries the bytes of both
    assert work["gate_up_gemm"][0] == "hbm" and work["down_gemm"] == ("fused", 0)
    d, I, n = 2048, 1408, 64 + 2
    weights = n * 3 * I * d * 2   # gate, up and down of every expert that received tokens
    streamed = work["gate_up_gemm"][1]
    assert weights < streamed < weights * 1.01
    # fewer active experts, fewer weight bytes
    assert bench.algorithmic_work(w, active_experts=10)["gate_up_gemm"][1] < work["gate_up_gemm"][1]


def test_source_digest_ignores_comments_and_whitespace_only():
    code = "int f(int x) {\n  return x + 1;  // add one\n}\n/* block\n comment */"
    same = "int f(int x){return x+1;}"
    other = "int f(int x){return x+2;}"
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)
    assert len(bench.csrc_digest()) == 40


def test_workload_description_names_the_layer_and_its_sizes():
    desc = bench.workload_desc(_shape("16b_prefill"), 4)
    assert desc["workload"].startswith("16b_prefill: T=16384 d=2048")
    assert desc["global_batch"] == 4 * 16384 and desc["parallelism"] == "dp4"


def _run_bench(args, env_extra=None):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env.update(env_extra or {})
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], cwd=root,
                       env=env, capture_output=True, text=True, timeout=600)
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    return p.returncode, [json.loads(l) for l in lines], p.stderr


def test_reference_arm_prints_one_contract_line_on_the_host():
    # the reference arm times the fp64 oracle on the host cores: no GPU involved
    rc, lines, err = _run_bench(["--impl", "reference", "--config", "tiny", "--steps", "2",
                                 "--warmup", "3"])
    assert rc == 0, err
    assert len(lines) == 1
    j = lines[0]
    assert j["impl"] == "reference" and j["unit"] == "tokens/s" and j["value"] > 0
    assert j["steps"] == 2 and j["warmup"] == 3 and j["n_gpus"] == 1
    assert j["higher_is_better"] is True and j["config"]["workload"].startswith("tiny:")
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    # under torchrun only rank 0 runs the oracle and prints
    rc, lines, err = _run_bench(["--impl", "reference", "--gpus", "2", "--config", "tiny",
                                 "--steps", "1", "--warmup", "3"], {"RANK": "1", "WORLD_SIZE": "2",
                                                    "LOCAL_RANK": "1"})
    assert rc == 0, err
    assert lines == []


def _bench(*argv, env=None):
    import subprocess
    import sys
    e = dict(os.environ)
    e.pop("WORLD_SIZE", None)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv], env=e,
                          capture_output=True, text=True, timeout=240)


def test_gpus_flag_launches_that_many_ranks():
    """`--gpus 2` outside a launcher starts two ranks (torchrun); on CPU the dry run takes
    the balance-loss exchange through gloo and rank 0 prints one line with n_gpus 2 and the
    global loss of both ranks' statistics."""
    import json

    import numpy as np

    from mixture_experts_layer_65_b200 import workloads as W
    p = _bench("--gpus", "2", "--dry-run", "--steps", "3", "--warmup", "3")
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads(l) for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["dry_run"] and line["value"] is None
    spec = W.CONFIGS["16b_prefill"]
    T, nr, K = spec["T"], spec["n_routed"], spec["top_k"]
    c = np.zeros(nr)
    ps = np.zeros(nr)
    for rank in range(2):   # the ranks' synthetic statistics, as bench.py draws them
        rng = np.random.default_rng(rank)
        c += rng.multinomial(T * K, np.full(nr, 1.0 / nr))
        ps += (rng.dirichlet(np.ones(nr)) * T).astype(np.float32)
    n = 2 * T
    assert line["global_tokens"] == n
    assert line["aux_loss"] == pytest.approx(spec["alpha1"] * np.sum((c / n) * (ps / n)), rel=1e-5)


def test_gpus_flag_must_match_the_launcher():
    p = _bench("--gpus", "1", "--dry-run", env={"WORLD_SIZE": "2"})
    assert p.returncode == 2
    assert "must agree" in p.stderr


def test_peak_regime_follows_the_sampled_clock():
    """Tensor-bound kernels are held against the burst peak unless the run was power-capped
    (sw_power_cap seen, median SM clock below 90% of the maximum, timed >= 0.5 s)."""
    burst = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1280.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.peak_regime(burst, 0.04) == "burst"
    assert bench.peak_regime(burst, 5.0) == "burst"
    assert bench.peak_regime(capped, 5.0) == "sustained"
    assert bench.peak_regime(capped, 0.04) == "burst"
    assert bench.peak_regime(None, 5.0) == "burst"
    assert bench.PEAK_KEY["burst"] == "bf16_tflops"


def test_kernel_timing_follows_the_timed_regions_clock_regime():
    """A burst-clock timed region takes the per-kernel pass measured before it (after a
    pause); a power-capped one the pass right after it; eager runs their own timed steps."""
    burst = ({"gate_up_gemm": 1.0}, 8, {"sm_mhz": 1965.0})
    post = ({"gate_up_gemm": 2.0}, 100, {"sm_mhz": 1200.0})
    ms, n, clk, text = bench.choose_kernel_timing("burst", False, burst, post)
    assert (ms, n, clk) == burst and "before the timed region" in text
    ms, n, clk, text = bench.choose_kernel_timing("sustained", False, burst, post)
    assert (ms, n, clk) == post and "right after" in text
    ms, n, clk, text = bench.choose_kernel_timing("burst", True, None, post)
    assert (ms, n, clk) == post and "over the timed steps" in text
    # the regime itself: power-capped only when timed long enough with the cap seen
    capped = {"sm_mhz": 1200.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.peak_regime(capped, 0.8) == "sustained"
    assert bench.peak_regime(capped, 0.05) == "burst"
    assert bench.peak_regime({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}, 2.0) == "burst"
