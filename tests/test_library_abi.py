"""The C-ABI library builds for sm_100a, loads without a GPU and exports every
entry point declared in include/ocrdec.h.  No compute is called here."""
import ctypes
import os
import re

import pytest

from speculative_moe_decoding_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ocrdec.h")


@pytest.fixture(scope="module")
def lib():
    from speculative_moe_decoding_b200 import build
    build.build(jobs=4)
    from speculative_moe_decoding_b200 import ocrdec
    return ocrdec


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = set(re.findall(r"\b(ocrdec_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib.lib, n), n


def test_no_unexpected_exports(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {n for n in exported if n.startswith("ocrdec_")}
    assert ours == set(declared_functions())


@pytest.mark.parametrize("dims", [synth.TINY, synth.FULL])
def test_manifest_matches_generator(lib, dims):
    cfg = lib.make_config(dims.as_dict(), 3, 1, 2048)
    got = lib.manifest(cfg)
    want = [shape for _, shape in synth.manifest(dims)]
    assert got == want
    assert lib.ocrdec_workspace_bytes(ctypes.byref(cfg)) > 0


def test_config_validation(lib):
    good = synth.TINY.as_dict()
    ctx = ctypes.c_void_p()
    cfg = lib.make_config(good, 3, 1, 256)
    assert lib.ocrdec_create(ctypes.byref(cfg), ctypes.byref(ctx)) == lib.OK
    lib.ocrdec_destroy(ctx)
    bad_cases = [
        dict(good, n_heads=3),             # heads * head_dim != d
        dict(good, top_k=9),               # top_k > n_experts
        dict(good, shared_ffn=64),         # shared width must equal expert width
        dict(good, vocab=4095),            # vocab multiple of 8
        dict(good, n_heads=8, head_dim=32),  # head_dim 64 or 128 only
        dict(good, d_model=2048, n_heads=32),  # at most 16 heads
        dict(good, d_model=192, n_heads=3),    # d_model a multiple of 128
        dict(good, n_experts=65),          # routed experts beyond the router block
        dict(good, n_shared=9),            # shared experts beyond the routing tables
        dict(good, top_k=0),               # sizes must be positive
        dict(good, d_model=2176, n_heads=17),  # d_model beyond 2048 (and > 16 heads)
        dict(good, d_model=1536, n_heads=12, head_dim=128),  # W_qkv rows of an attention CTA beyond shared memory
        dict(good, n_dense_first=3),       # more dense layers than layers
        dict(good, n_dense_first=1, dense_ffn=100),  # dense width a multiple of 64
        dict(good, expert_ffn=96, shared_ffn=96),    # expert width a multiple of 64
        dict(good, rms_eps=0.0),           # eps must be positive
        dict(good, rope_theta=1.0),        # theta must exceed 1
    ]
    for bad in bad_cases:
        cfg = lib.make_config(bad, 3, 1, 256)
        assert lib.ocrdec_create(ctypes.byref(cfg), ctypes.byref(ctx)) == lib.EINVAL
    cfg = lib.make_config(good, 4, 1, 256)  # max_k > 3
    assert lib.ocrdec_create(ctypes.byref(cfg), ctypes.byref(ctx)) == lib.EINVAL
    cfg = lib.make_config(good, 3, 3, 256)  # batch * (k+1) rows beyond one pass
    assert lib.ocrdec_create(ctypes.byref(cfg), ctypes.byref(ctx)) == lib.EINVAL
    cfg = lib.make_config(good, 3, 1, 8200)  # kv_capacity beyond 8192
    assert lib.ocrdec_create(ctypes.byref(cfg), ctypes.byref(ctx)) == lib.EINVAL


def test_calls_before_setup_fail_cleanly(lib):
    ctx = ctypes.c_void_p()
    cfg = lib.make_config(synth.TINY.as_dict(), 3, 1, 256)
    assert lib.ocrdec_create(ctypes.byref(cfg), ctypes.byref(ctx)) == lib.OK
    try:
        assert lib.ocrdec_step(ctx, 1, 0, None, None, None) in (lib.ESTATE, lib.EINVAL)
        assert lib.ocrdec_prefill(ctx, 0, None, 0, None, 0, None, None) == lib.ESTATE
        assert lib.ocrdec_draft(ctx, 1, 1, None, None) == lib.ESTATE
        assert lib.ocrdec_bind_workspace(ctx, None, 0, None) == lib.EINVAL
        assert lib.ocrdec_strerror(lib.ECAPACITY) == b"KV capacity exceeded"
    finally:
        lib.ocrdec_destroy(ctx)


def test_op_argument_checks(lib):
    """The single-kernel entry points reject widths that are not whole 64-column
    chunks or exceed 2048, and row counts outside 1..8, before touching the GPU."""
    p = ctypes.c_void_p(256)  # never dereferenced: validation comes first
    for R, N, K in [(1, 64, 4000), (1, 64, 1000), (0, 64, 256), (9, 64, 256), (1, 0, 256), (1, 64, 32)]:
        assert lib.ocrdec_op_norm_gemv(p, p, p, ctypes.c_float(1e-6), R, N, K, p, p, None) == lib.EINVAL
        assert lib.ocrdec_op_lm_argmax(p, p, p, ctypes.c_float(1e-6), R, N, K, p, None, p, None) == lib.EINVAL


def test_binding_checks_op_arguments_before_the_abi():
    """The op wrappers reject wrong dtypes, shapes and layouts (and host
    tensors) before a pointer crosses the ABI."""
    import torch
    from speculative_moe_decoding_b200 import ocrdec
    W = torch.zeros(64, 256, dtype=torch.int16)
    x = torch.zeros(2, 256)
    g = torch.zeros(256, dtype=torch.bfloat16)
    y = torch.zeros(2, 64)
    tok = torch.zeros(2, dtype=torch.int32)
    sc = torch.zeros(ocrdec.ocrdec_op_scratch_bytes(), dtype=torch.uint8)
    small = torch.zeros(16, dtype=torch.uint8)
    bad = [
        (lambda: ocrdec.op_norm_gemv(W.float(), x, g, 1e-6, y, sc), "W: dtype"),
        (lambda: ocrdec.op_norm_gemv(W, x.double(), g, 1e-6, y, sc), "x: dtype"),
        (lambda: ocrdec.op_norm_gemv(W, x, g[:128], 1e-6, y, sc), "g: shape"),
        (lambda: ocrdec.op_norm_gemv(W, x, g, 1e-6, y[:, :32].contiguous(), sc), "y: shape"),
        (lambda: ocrdec.op_norm_gemv(W, x, g, 1e-6, torch.zeros(64, 2).t(), sc), "y: must be contiguous"),
        (lambda: ocrdec.op_lm_argmax(W, x, g, 1e-6, tok.long(), None, sc), "tok: dtype"),
        (lambda: ocrdec.op_lm_argmax_static(W, x, g, 1e-6, tok, torch.zeros(2, 63)), "logits: shape"),
        (lambda: ocrdec.op_norm_gemv(W, x, g, 1e-6, y, small), "scratch: 16 bytes, need at least"),
        (lambda: ocrdec.op_lm_argmax(W, x, g, 1e-6, tok, None, small), "scratch: 16 bytes, need at least"),
        (lambda: ocrdec.op_norm_gemv(W, x, g, 1e-6, y.to("meta"), sc), "y: on meta, but x is on cpu"),
        (lambda: ocrdec.op_lm_argmax(W.to("meta"), x, g, 1e-6, tok, None, sc), "W: on meta"),
        (lambda: ocrdec.op_lm_argmax_static(W, x, g, 1e-6, tok, torch.zeros(2, 64, device="meta")), "logits: on meta"),
        (lambda: ocrdec.op_norm_gemv(W, x, g, 1e-6, y, sc), "must be a CUDA tensor"),
    ]
    for call, msg in bad:
        with pytest.raises(ValueError, match=msg):
            call()
