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
