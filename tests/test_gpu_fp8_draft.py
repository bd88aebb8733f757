"""The cheaper draft argmax (a variant the pages do not describe): the draft
reads an e4m3 copy of the LM head.  Checked here:

* the copy: every byte decodes (e4m3, written out below from the format's
  definition) to the bf16 weight times the row's scale within e4m3 rounding,
  and each row's largest magnitude maps to 448;
* the draft's logits with the e4m3 head against its logits with the bf16
  head from the same state, within the quantisation error;
* losslessness: verification is greedy with the bf16 head, so k = 3 with the
  e4m3 draft commits exactly the library's own k = 0 tokens (model page:
  bit-identical to plain autoregressive decoding)."""
import numpy as np
import pytest

from speculative_moe_decoding_b200 import synth

from .gpu_util import gpu_decode, make_decoder, to_dev

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS["tiny"]


def e4m3_to_float(b: np.ndarray) -> np.ndarray:
    """e4m3 bytes -> float64: sign, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent 0 is subnormal (m/8 * 2^-6); 0x7f / 0xff are NaN (no infinities)."""
    b = b.astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    v = np.where((b & 0x7F) == 0x7F, np.nan, v)
    return s * v


def test_e4m3_decoder_special_values():
    # 0x7e = 1.75 * 2^8 = 448 (largest finite), 0x38 = 1.0, 0x01 = 2^-9 (smallest subnormal)
    np.testing.assert_array_equal(e4m3_to_float(np.array([0x7E, 0x38, 0x01, 0x00, 0xB8, 0x08])),
                                  [448.0, 1.0, 2.0 ** -9, 0.0, -1.0, 2.0 ** -6])


@pytest.fixture(scope="module")
def tiny_bits():
    bits, _ = synth.make_weights(synth.TINY, W.weight_seed, workers=1)
    return bits


def test_quantised_head_matches_the_bf16_head(tiny_bits):
    import torch
    from oracle.decoder import bf16_bits_to_f32
    m = synth.TINY
    dec = make_decoder(m, tiny_bits, max_k=3, max_batch=1, kv_capacity=256)
    try:
        buf = dec.set_draft_head_fp8(True)
        torch.cuda.synchronize()
        V, d = m.vocab, m.d_model
        raw = buf.cpu().numpy()
        w8 = raw[:V * d].reshape(V, d)
        off = ((V * d + 255) // 256) * 256
        inv = raw[off:off + 4 * V].view(np.float32)
    finally:
        dec.close()
    Wf = bf16_bits_to_f32(tiny_bits["lm_head"]).astype(np.float64)
    amax = np.abs(Wf).max(axis=1)
    np.testing.assert_allclose(inv, amax / 448.0, rtol=1e-6)
    q = e4m3_to_float(w8)
    assert not np.isnan(q).any()
    scaled = Wf * (448.0 / amax)[:, None]
    # round to nearest: half a unit of the last place (2^-4 relative for
    # normals, 2^-10 absolute for subnormals)
    ulp = np.where(np.abs(scaled) >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(scaled), 1e-30))) - 3),
                   2.0 ** -9)
    assert np.all(np.abs(q - scaled) <= 0.5 * ulp + 1e-12)
    assert np.all(np.abs(q).max(axis=1) == 448.0)


def test_draft_logits_with_the_e4m3_head(tiny_bits):
    import torch
    m = synth.TINY
    inp = synth.make_inputs(m, W.input_seed, W.n_visual, W.n_prompt)
    dec = make_decoder(m, tiny_bits, max_k=3, max_batch=1, kv_capacity=256)
    try:
        vis, prm = to_dev(inp)
        dec.set_forced_acceptance(None, None, None, ())
        dec.prefill(0, vis, prm)
        for _ in range(3):
            dec.verify_commit(1, 0)
        # the draft from the same slot state, once per head (the draft only
        # rewrites its own cache rows with the same values)
        taps = []
        for fp8 in (False, True):
            dec.set_draft_head_fp8(fp8)
            t = torch.zeros((3, 1, m.vocab), dtype=torch.float32, device="cuda")
            dec.set_draft_taps(t)
            props = dec.draft(1, 1)[:1].clone()
            dec.set_draft_taps(None)
            torch.cuda.synchronize()
            taps.append((t[0, 0].cpu().numpy(), int(props[0].item())))
        assert dec.status() == 0
    finally:
        dec.close()
    (lb, pb), (l8, p8) = taps
    assert pb == int(np.argmax(lb)) and p8 == int(np.argmax(l8))  # each head's token is its own argmax
    err = np.abs(l8 - lb)
    # e4m3 weights (2^-4 relative) and activation parts: a few percent of the logit scale
    assert err.max() <= 0.08 * np.abs(lb).max(), (err.max(), np.abs(lb).max())
    assert err.mean() <= 0.03 * np.abs(lb).mean()
    assert np.corrcoef(l8, lb)[0, 1] > 0.995


@pytest.mark.parametrize("k", [1, 3])
def test_speculative_with_e4m3_draft_is_bit_identical_to_k0(tiny_bits, k):
    m = synth.TINY
    inp = synth.make_inputs(m, W.input_seed, W.n_visual, W.n_prompt)
    dec = make_decoder(m, tiny_bits, max_k=3, max_batch=1, kv_capacity=256)
    try:
        ref, _, _ = gpu_decode(dec, inp, 0, W.n_generate)
        dec.set_draft_head_fp8(True)
        got, st, _ = gpu_decode(dec, inp, k, W.n_generate)
        assert dec.status() == 0
    finally:
        dec.close()
    assert np.array_equal(got, ref)


def test_bench_workload_with_e4m3_draft_is_bit_identical_to_k0(full_bits):
    import torch
    m = synth.FULL
    w = synth.WORKLOADS["full_spec"]
    inp = synth.make_inputs(m, w.input_seed, w.n_visual, w.n_prompt)
    C = w.n_visual + w.n_prompt
    n_gen, n_ref = 64, 128
    dec = make_decoder(m, full_bits, max_k=3, max_batch=1, kv_capacity=C + n_ref + 64)
    try:
        k0, _, _ = gpu_decode(dec, inp, 0, n_ref)
        ref_hist = dec.history(0, 0, C + n_ref).clone()
        dec.set_draft_head_fp8(True)
        real, _, _ = gpu_decode(dec, inp, 3, n_gen)
        tab = synth.make_forced_tables(w.stream_seed, C + n_ref, m.vocab, 3, w.accept_p)
        forced = (ref_hist, torch.from_numpy(tab.u).cuda(), torch.from_numpy(tab.r).cuda(), tab.p)
        got, st, _ = gpu_decode(dec, inp, 3, n_gen, forced=forced)
        assert dec.status() == 0
    finally:
        dec.close()
    assert np.array_equal(real, k0[:n_gen])
    assert np.array_equal(got, k0[:n_gen])
    assert st.tau_sum / st.steps > 2.0
