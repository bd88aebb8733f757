"""The LM-head argmax entry point that allocates nothing (library-owned static
scratch) against the caller-scratch entry point, on the same inputs, two calls
in a row.  Kept in its own file, collected last; it needs no fixture state, so
it passes alone in a fresh process as well as after the other tests."""
import numpy as np
import pytest

from speculative_moe_decoding_b200 import synth


@pytest.mark.gpu
@pytest.mark.parametrize("R,N,K", [(1, 4096, 256), (4, 129280, 1280)])
def test_static_scratch_matches_caller_scratch(R, N, K):
    import torch
    from speculative_moe_decoding_b200 import ocrdec
    rng = np.random.default_rng(7 * N + R)
    Wb = synth.f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * 0.02)
    gb = synth.f32_to_bf16_bits(1.0 + 0.1 * rng.standard_normal(K, dtype=np.float32))
    x = rng.standard_normal((R, K), dtype=np.float32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    W, g, xd = t(Wb.view(np.int16)), t(gb.view(np.int16)), t(x)

    tok_ref = torch.empty(R, dtype=torch.int32, device="cuda")
    lg_ref = torch.empty((R, N), dtype=torch.float32, device="cuda")
    ocrdec.op_lm_argmax(W, xd, g, 1e-6, tok_ref, lg_ref, ocrdec.op_scratch())
    torch.cuda.synchronize()
    for _ in range(2):  # two calls in a row reuse the same static scratch
        tok = torch.full((R,), -1, dtype=torch.int32, device="cuda")
        lg = torch.zeros((R, N), dtype=torch.float32, device="cuda")
        ocrdec.op_lm_argmax_static(W, xd, g, 1e-6, tok, lg)
        torch.cuda.synchronize()
        # same kernel, same fixed reduction order: bit for bit the same logits
        assert np.array_equal(lg.cpu().numpy().view(np.uint32), lg_ref.cpu().numpy().view(np.uint32))
        assert np.array_equal(tok.cpu().numpy(), tok_ref.cpu().numpy())


def test_static_scratch_size_is_exported():
    from speculative_moe_decoding_b200 import ocrdec
    assert ocrdec.ocrdec_op_static_scratch_bytes() == 64 * 1024
