"""Helpers for the GPU tests: build a library decoder from the seeded weights
and run decodes through the C ABI."""
from __future__ import annotations

import numpy as np

from speculative_moe_decoding_b200 import synth


def make_decoder(dims: synth.ModelDims, bits, max_k=3, max_batch=1, kv_capacity=512):
    from speculative_moe_decoding_b200 import build
    build.build(jobs=4)
    from speculative_moe_decoding_b200 import ocrdec
    names = [n for n, _ in synth.manifest(dims)]
    return ocrdec.Decoder(dims.as_dict(), bits, names, max_k=max_k, max_batch=max_batch, kv_capacity=kv_capacity)


def to_dev(inputs: synth.SeqInputs):
    import torch
    vis = torch.from_numpy(inputs.visual).cuda()
    prm = torch.from_numpy(inputs.prompt).cuda()
    return vis, prm


def gpu_decode(dec, inputs: synth.SeqInputs, k: int, n_gen: int, graph: bool = True, forced=None,
               record_proposals: bool = False, chunk_steps: int = 8):
    """Prefill slot 0, then run steps until n_gen tokens are generated.  Returns
    (tokens [n_gen], taus, proposals-per-step or None)."""
    import torch
    vis, prm = to_dev(inputs)
    C = inputs.visual.shape[0] + inputs.prompt.shape[0]
    dec.set_forced_acceptance(*forced) if forced is not None else dec.set_forced_acceptance(None, None, None, ())
    dec.prefill(0, vis, prm)
    taus, props_log = [], []
    while True:
        st = dec.stats(0)
        assert dec.status() == 0, dec.status()
        if st.n_generated >= n_gen:
            break
        for _ in range(chunk_steps):
            if record_proposals or not graph:
                if k > 0:
                    p = dec.draft(1, k)
                    if forced is not None:
                        raise ValueError("eager path with forced acceptance is not exercised here")
                    if record_proposals:
                        props_log.append(p[:k].cpu().numpy().copy())
                    dec.verify_commit(1, k, p)
                else:
                    dec.verify_commit(1, 0, None)
            else:
                dec.step(1, k)
            if record_proposals:
                taus.append(int(dec.n_committed[0].item()))
    torch.cuda.synchronize()
    toks = dec.history(0, C, n_gen).cpu().numpy().astype(np.int64)
    st = dec.stats(0)
    return toks, st, (props_log if record_proposals else None)
