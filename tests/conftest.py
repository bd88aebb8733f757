import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def tiny_weights():
    from speculative_moe_decoding_b200 import synth
    bits, f32 = synth.make_weights(synth.TINY, 0, keep_f32=True, workers=1)
    return bits, f32


@pytest.fixture(scope="session")
def tiny_inputs():
    from speculative_moe_decoding_b200 import synth
    w = synth.WORKLOADS["tiny"]
    return synth.make_inputs(synth.TINY, w.input_seed, w.n_visual, w.n_prompt)


@pytest.fixture(scope="session")
def full_bits():
    """bf16 weight bits of the full-size model (the benchmark's seed), made once
    per session and shared by the full-size GPU tests."""
    from speculative_moe_decoding_b200 import synth
    bits, _ = synth.make_weights(synth.FULL, synth.WORKLOADS["full_spec"].weight_seed)
    return bits
