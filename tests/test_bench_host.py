"""Host-side logic of bench.py's CPU legs on tiny inputs (no GPU).

The cpu_baseline leg sizes its sample by timing the oracle, so on a fast host it can ask for
more token rows than a linear has; the sampled rows must then wrap around instead of indexing
past the activations.
"""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_host_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _tiny_linears():
    from bit_weight_quantization_wq_b200 import synth
    return synth.flux_linears(M=8, rank=4, shapes=[(256, 256), (384, 256), (256, 512)])


def test_oracle_sample_wraps_token_rows():
    bench = _load_bench()
    lins = _tiny_linears()
    # 3 linears x 40 token rows with offsets 0, 17, 34 against M = 8: every index wraps
    flops, params, secs = bench.oracle_sample(lins, 40, 128)
    assert params == sum(min(128, lin["N"]) * lin["K"] for lin in lins)
    assert flops > 0 and secs >= 0


def test_cpu_baseline_caps_rows_on_a_fast_host():
    bench = _load_bench()
    out = bench.cpu_baseline(_tiny_linears(), budget_s=0.5)
    assert out["kind"] == "oracle" and out["unit"] == "TFLOP/s"
    assert out["value"] > 0 and out["cores"] >= 1
