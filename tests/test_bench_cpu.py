"""The CPU side of bench.py: the oracle sample behind cpu_baseline and the
reference arm (tiny model, short budgets), and the step byte model."""
import bench
from speculative_moe_decoding_b200 import synth


def test_oracle_sample_and_variants():
    bits, _ = synth.make_weights(synth.TINY, synth.WORKLOADS["tiny"].weight_seed, workers=1)
    tps, desc, used, steps, dt = bench.run_oracle_sample(synth.TINY, 3, bits, budget_s=0.3)
    assert tps > 0 and steps > 0 and dt >= 0.3 and used >= 1
    assert "k=3" in desc and "repetitions" in desc
    var = bench.oracle_variants(synth.TINY, 3, bits, budget_s=0.2)
    assert [v["k"] for v in var] == [0, 3]
    assert var[1]["threads"] == 1
    assert all(v["value"] and v["value"] > 0 for v in var)


def test_step_bytes_dense_set():
    # the dense set of the full model: attention + layer-0 FFN + shared experts
    # + routers + LM head = 694,026,240 bytes; routed experts add 6,881,280 B each
    m = synth.FULL
    union0, dep0 = bench.step_bytes(m, 0, 0.0, 0.0)
    assert union0 == dep0 == 694_026_240
    union1, _ = bench.step_bytes(m, 0, 1.0, 0.0)
    assert union1 - union0 == 11 * 6_881_280


def test_oracle_sample_exact_steps():
    # the reference arm: W untimed steps, then exactly K timed ones
    bits, _ = synth.make_weights(synth.TINY, synth.WORKLOADS["tiny"].weight_seed, workers=1)
    tps, desc, used, steps, dt = bench.run_oracle_sample(synth.TINY, 3, bits, timed_steps=7, warm_steps=2)
    assert steps == 7 and tps > 0 and dt > 0


def test_profiled_traffic_hash_and_scaling(tmp_path, monkeypatch):
    import hashlib
    src = tmp_path / "kernel.cuh"
    src.write_text("// kernel source\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles").mkdir()
    prof = tmp_path / "profiles" / "k.md"
    prof.write_text("# capture\n\n    traffic_bytes_per_launch: 1030\n    algorithmic_bytes_per_launch: 1000\n"
                    f"    source_sha256: {digest}\n    source_files: kernel.cuh\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k.md") == 1030
    assert abs(bench.profiled_traffic("k.md", 5000) - 5150) < 1e-9  # the ratio, scaled to this launch
    assert bench.profiled_traffic("missing.md") is None
    src.write_text("// kernel source, changed\n")
    assert bench.profiled_traffic("k.md") is None  # counters of an older kernel are not reported
