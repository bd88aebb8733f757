"""ctypes binding of libocrdec.so (C ABI in include/ocrdec.h).

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  Importing this
module raises if the library has not been built - there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libocrdec.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m speculative_moe_decoding_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

OK, EINVAL, ENOMEM, ECUDA, ECAPACITY, ETIMEOUT, ESTATE = range(7)

_i32, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class Config(ctypes.Structure):
    _fields_ = [(n, _i32) for n in (
        "d_model", "n_layers", "n_heads", "head_dim", "n_dense_first", "n_experts", "n_shared", "top_k",
        "expert_ffn", "shared_ffn", "dense_ffn", "draft_ffn", "vocab", "max_k", "max_batch", "kv_capacity")] + [
        ("rope_theta", _f32), ("rms_eps", _f32)]


class SlotStats(ctypes.Structure):
    _fields_ = [("kv_len", _i32), ("n_context", _i32), ("n_generated", _i32), ("bonus", _i32), ("steps", _i32),
                ("tau_sum", _i32), ("accepted_hist", _i32 * 4)]


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


ocrdec_create = _sig("ocrdec_create", _i32, ctypes.POINTER(Config), ctypes.POINTER(_vp))
ocrdec_destroy = _sig("ocrdec_destroy", None, _vp)
ocrdec_weight_count = _sig("ocrdec_weight_count", _i32, ctypes.POINTER(Config))
ocrdec_weight_info = _sig("ocrdec_weight_info", _i32, ctypes.POINTER(Config), _i32,
                          ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(_i32))
ocrdec_workspace_bytes = _sig("ocrdec_workspace_bytes", _sz, ctypes.POINTER(Config))
ocrdec_bind_workspace = _sig("ocrdec_bind_workspace", _i32, _vp, _vp, _sz, _vp)
ocrdec_load_weights = _sig("ocrdec_load_weights", _i32, _vp, ctypes.POINTER(_vp), _i32)
ocrdec_prefill = _sig("ocrdec_prefill", _i32, _vp, _i32, _vp, _i32, _vp, _i32, _vp, _vp)
ocrdec_draft = _sig("ocrdec_draft", _i32, _vp, _i32, _i32, _vp, _vp)
ocrdec_verify_commit = _sig("ocrdec_verify_commit", _i32, _vp, _i32, _i32, _vp, _vp, _vp, _vp)
ocrdec_step = _sig("ocrdec_step", _i32, _vp, _i32, _i32, _vp, _vp, _vp)
ocrdec_step_host = _sig("ocrdec_step_host", _i32, _vp, _i32, _i32, _vp, _vp, _vp)
ocrdec_set_forced_acceptance = _sig("ocrdec_set_forced_acceptance", _i32, _vp, _vp, _vp, _vp, _i32, _vp)
ocrdec_get_status = _sig("ocrdec_get_status", _i32, _vp, ctypes.POINTER(_i32), _vp)
ocrdec_clear_status = _sig("ocrdec_clear_status", _i32, _vp, _vp)
ocrdec_get_slot_stats = _sig("ocrdec_get_slot_stats", _i32, _vp, _i32, ctypes.POINTER(SlotStats), _vp)
ocrdec_token_history = _sig("ocrdec_token_history", _i32, _vp, _i32, ctypes.POINTER(_vp))
ocrdec_get_counters = _sig("ocrdec_get_counters", _i32, _vp, ctypes.POINTER(_i32), _i32, _vp)
ocrdec_reset_counters = _sig("ocrdec_reset_counters", _i32, _vp, _vp)
ocrdec_step_kernel_count = _sig("ocrdec_step_kernel_count", _i32, _vp, _i32, _i32, _vp, _vp, ctypes.POINTER(_i32))
ocrdec_set_debug_taps = _sig("ocrdec_set_debug_taps", _i32, _vp, _vp, _vp)
ocrdec_set_draft_taps = _sig("ocrdec_set_draft_taps", _i32, _vp, _vp)
ocrdec_set_trace = _sig("ocrdec_set_trace", _i32, _vp, _i32, _vp)
ocrdec_draft_head_fp8_bytes = _sig("ocrdec_draft_head_fp8_bytes", _sz, ctypes.POINTER(Config))
ocrdec_set_draft_head_fp8 = _sig("ocrdec_set_draft_head_fp8", _i32, _vp, _vp, _sz, _vp)
ocrdec_replay_moe_ffn = _sig("ocrdec_replay_moe_ffn", _i32, _vp, _i32, _i32, _i32, _i32, _vp)
ocrdec_read_trace = _sig("ocrdec_read_trace", _i32, _vp, _vp, _i32, ctypes.POINTER(_i32), _vp)

TRACE_DTYPE = np.dtype([("t0", "<u8"), ("d1", "<u4"), ("d2", "<u4"), ("dt", "<u4"), ("tag", "<u2"),
                        ("sm", "<u2")])
ocrdec_strerror = _sig("ocrdec_strerror", ctypes.c_char_p, _i32)
ocrdec_op_scratch_bytes = _sig("ocrdec_op_scratch_bytes", _sz)
ocrdec_op_norm_gemv = _sig("ocrdec_op_norm_gemv", _i32, _vp, _vp, _vp, _f32, _i32, _i32, _i32, _vp, _vp, _vp)
ocrdec_op_lm_argmax = _sig("ocrdec_op_lm_argmax", _i32, _vp, _vp, _vp, _f32, _i32, _i32, _i32, _vp, _vp, _vp, _vp)
ocrdec_op_lm_argmax_static = _sig("ocrdec_op_lm_argmax_static", _i32, _vp, _vp, _vp, _f32, _i32, _i32, _i32, _vp,
                                  _vp, _vp)
ocrdec_op_static_scratch_bytes = _sig("ocrdec_op_static_scratch_bytes", _sz)


class OcrdecError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {ocrdec_strerror(code).decode()} ({code})")
        self.code = code


def check(code: int, where: str) -> None:
    if code != OK:
        raise OcrdecError(code, where)


def make_config(dims: dict, max_k: int = 3, max_batch: int = 1, kv_capacity: int = 2048) -> Config:
    c = Config()
    for k in ("d_model", "n_layers", "n_heads", "head_dim", "n_dense_first", "n_experts", "n_shared", "top_k",
              "expert_ffn", "shared_ffn", "dense_ffn", "draft_ffn", "vocab"):
        setattr(c, k, int(dims[k]))
    c.max_k, c.max_batch, c.kv_capacity = max_k, max_batch, kv_capacity
    c.rope_theta, c.rms_eps = float(dims["rope_theta"]), float(dims["rms_eps"])
    return c


def manifest(cfg: Config):
    n = ocrdec_weight_count(ctypes.byref(cfg))
    if n < 0:
        raise OcrdecError(-n, "ocrdec_weight_count")
    out = []
    dims = (ctypes.c_int64 * 3)()
    nd = _i32()
    for i in range(n):
        check(ocrdec_weight_info(ctypes.byref(cfg), i, dims, ctypes.byref(nd)), "ocrdec_weight_info")
        out.append(tuple(dims[j] for j in range(nd.value)))
    return out


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class Decoder:
    """One library context with its workspace and borrowed weights (torch CUDA tensors)."""

    def __init__(self, dims: dict, weight_bits: Dict[str, np.ndarray], names: Sequence[str], *, max_k: int = 3,
                 max_batch: int = 1, kv_capacity: int = 2048, device: str = "cuda"):
        import torch
        self.torch = torch
        self.cfg = make_config(dims, max_k, max_batch, kv_capacity)
        self.dims = dict(dims)
        self.max_k, self.max_batch = max_k, max_batch
        shapes = manifest(self.cfg)
        if len(shapes) != len(names):
            raise ValueError(f"manifest has {len(shapes)} tensors, got {len(names)} names")
        self.weights = []
        for name, shp in zip(names, shapes):
            a = weight_bits[name]
            if tuple(a.shape) != tuple(shp) or a.dtype != np.uint16:
                raise ValueError(f"{name}: expected uint16 {shp}, got {a.dtype} {a.shape}")
            self.weights.append(torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device))
        ctx = _vp()
        check(ocrdec_create(ctypes.byref(self.cfg), ctypes.byref(ctx)), "ocrdec_create")
        self.ctx = ctx
        nbytes = ocrdec_workspace_bytes(ctypes.byref(self.cfg))
        self.workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.workspace.data_ptr()) % 256
        self.ws_ptr = self.workspace.data_ptr() + off
        check(ocrdec_bind_workspace(self.ctx, self.ws_ptr, nbytes, _stream(None)), "ocrdec_bind_workspace")
        ptrs = (_vp * len(self.weights))(*[w.data_ptr() for w in self.weights])
        check(ocrdec_load_weights(self.ctx, ptrs, len(self.weights)), "ocrdec_load_weights")
        self._i32 = lambda n: torch.empty(n, dtype=torch.int32, device=device)
        self.committed = self._i32(max_batch * (max_k + 1))
        self.n_committed = self._i32(max_batch)
        self.proposals = self._i32(max_batch * max(1, max_k))
        self._forced = None
        self._taps = None

    def close(self):
        if getattr(self, "ctx", None):
            ocrdec_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- decode path -----------------------------------------------------
    def prefill(self, slot: int, visual, prompt, stream=None):
        """visual: float32 CUDA tensor [n_visual, d]; prompt: int32 CUDA tensor.  Returns a 1-element
        int32 CUDA tensor holding the first generated token."""
        torch = self.torch
        if visual is not None:
            _need(visual, "visual", (torch.float32,), (int(visual.shape[0]), int(self.dims["d_model"])))
        if prompt is not None:
            _need(prompt, "prompt", (torch.int32,), (int(prompt.numel()),))
        for name, t in (("visual", visual), ("prompt", prompt)):
            if t is not None and t.device != self.workspace.device:
                raise ValueError(f"{name}: on {t.device}, but the decoder lives on {self.workspace.device}")
        out = self._i32(1)
        check(ocrdec_prefill(self.ctx, slot, _ptr(visual), int(visual.shape[0]) if visual is not None else 0,
                             _ptr(prompt), int(prompt.shape[0]) if prompt is not None else 0, out.data_ptr(),
                             _stream(stream)), "ocrdec_prefill")
        return out

    def draft(self, batch: int, k: int, proposals=None, stream=None):
        p = self.proposals if proposals is None else proposals
        check(ocrdec_draft(self.ctx, batch, k, p.data_ptr(), _stream(stream)), "ocrdec_draft")
        return p

    def verify_commit(self, batch: int, k: int, proposals=None, stream=None):
        check(ocrdec_verify_commit(self.ctx, batch, k, _ptr(proposals) if k > 0 else None,
                                   self.committed.data_ptr(), self.n_committed.data_ptr(), _stream(stream)),
              "ocrdec_verify_commit")
        return self.committed, self.n_committed

    def step(self, batch: int, k: int, stream=None):
        check(ocrdec_step(self.ctx, batch, k, self.committed.data_ptr(), self.n_committed.data_ptr(),
                          _stream(stream)), "ocrdec_step")
        return self.committed, self.n_committed

    def step_host(self, batch: int, k: int, host_committed: np.ndarray, host_n: np.ndarray, stream=None):
        check(ocrdec_step_host(self.ctx, batch, k, host_committed.ctypes.data, host_n.ctypes.data,
                               _stream(stream)), "ocrdec_step_host")

    def set_forced_acceptance(self, ref, u, alt, p: Sequence[float]):
        """ref: int32 CUDA [n_pos]; u: float32 CUDA [n_pos, max_k]; alt: int32 CUDA [n_pos, max_k]."""
        if ref is None:
            self._forced = None
            check(ocrdec_set_forced_acceptance(self.ctx, None, None, None, 0, None), "ocrdec_set_forced_acceptance")
            return
        pa = (_f32 * 3)(*(list(p) + [0.0, 0.0, 0.0])[:3])
        self._forced = (ref, u, alt, pa)
        check(ocrdec_set_forced_acceptance(self.ctx, ref.data_ptr(), u.data_ptr(), alt.data_ptr(),
                                           int(ref.shape[0]), ctypes.cast(pa, _vp)), "ocrdec_set_forced_acceptance")

    # ---- state -------------------------------------------------------------
    def status(self, stream=None) -> int:
        s = _i32()
        check(ocrdec_get_status(self.ctx, ctypes.byref(s), _stream(stream)), "ocrdec_get_status")
        return s.value

    def clear_status(self, stream=None):
        check(ocrdec_clear_status(self.ctx, _stream(stream)), "ocrdec_clear_status")

    def stats(self, slot: int = 0, stream=None) -> SlotStats:
        st = SlotStats()
        check(ocrdec_get_slot_stats(self.ctx, slot, ctypes.byref(st), _stream(stream)), "ocrdec_get_slot_stats")
        return st

    def history(self, slot: int, start: int, n: int):
        """Committed tokens at positions start..start+n-1 (a CUDA int32 view)."""
        p = _vp()
        check(ocrdec_token_history(self.ctx, slot, ctypes.byref(p)), "ocrdec_token_history")
        torch = self.torch
        base = p.value - self.ws_ptr
        ws = self.workspace[(self.ws_ptr - self.workspace.data_ptr()):]
        return ws[base + 4 * start: base + 4 * (start + n)].view(torch.int32)

    def counters(self, stream=None):
        out = (_i32 * 2)()
        check(ocrdec_get_counters(self.ctx, out, 2, _stream(stream)), "ocrdec_get_counters")
        return out[0], out[1]

    def reset_counters(self, stream=None):
        check(ocrdec_reset_counters(self.ctx, _stream(stream)), "ocrdec_reset_counters")

    def step_kernel_count(self, batch: int, k: int) -> int:
        n = _i32()
        check(ocrdec_step_kernel_count(self.ctx, batch, k, self.committed.data_ptr(), self.n_committed.data_ptr(),
                                       ctypes.byref(n)), "ocrdec_step_kernel_count")
        return n.value

    def set_trace(self, enable: bool, stream=None):
        check(ocrdec_set_trace(self.ctx, 1 if enable else 0, _stream(stream)), "ocrdec_set_trace")

    def read_trace(self, max_records: int = 1 << 19, stream=None) -> np.ndarray:
        buf = np.zeros(max_records, dtype=TRACE_DTYPE)
        n = _i32()
        check(ocrdec_read_trace(self.ctx, buf.ctypes.data, max_records, ctypes.byref(n), _stream(stream)),
              "ocrdec_read_trace")
        return buf[:min(n.value, max_records)]

    def replay_moe_ffn(self, batch: int, k: int, first_layer: int, n_layers: int, stream=None):
        """Timing hook: the MoE FFN kernels of verifier layers first_layer.. again, on the last
        (batch, k) pass's rows and routing."""
        check(ocrdec_replay_moe_ffn(self.ctx, batch, k, first_layer, n_layers, _stream(stream)),
              "ocrdec_replay_moe_ffn")

    def set_draft_head_fp8(self, enable: bool = True, stream=None):
        """Variant: the draft's argmax over an e4m3 copy of the LM head (verification unchanged).
        Returns the (uint8) buffer holding the copy and its inverse row scales, or None."""
        torch = self.torch
        if not enable:
            self._head8 = None
            check(ocrdec_set_draft_head_fp8(self.ctx, None, 0, _stream(stream)), "ocrdec_set_draft_head_fp8")
            return None
        n = int(ocrdec_draft_head_fp8_bytes(ctypes.byref(self.cfg)))
        buf = torch.empty(n + 256, dtype=torch.uint8, device=self.workspace.device)
        off = (-buf.data_ptr()) % 256
        self._head8 = buf[off:off + n]
        check(ocrdec_set_draft_head_fp8(self.ctx, self._head8.data_ptr(), n, _stream(stream)),
              "ocrdec_set_draft_head_fp8")
        return self._head8

    def set_draft_taps(self, logits=None):
        self._dtaps = logits
        check(ocrdec_set_draft_taps(self.ctx, _ptr(logits)), "ocrdec_set_draft_taps")

    def set_debug_taps(self, hidden=None, logits=None):
        self._taps = (hidden, logits)
        check(ocrdec_set_debug_taps(self.ctx, _ptr(hidden), _ptr(logits)), "ocrdec_set_debug_taps")


# ---- single-kernel entry points ---------------------------------------------
def op_scratch(device="cuda"):
    import torch
    return torch.zeros(ocrdec_op_scratch_bytes(), dtype=torch.uint8, device=device)


def _need(t, name, dtypes, shape=None, cuda=True):
    """Argument checks before a pointer crosses the ABI: a torch tensor of one
    of the dtypes, the given shape, contiguous and (cuda) on a CUDA device."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor, got {type(t).__name__}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {', '.join(map(str, dtypes))}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")


def _bf16_types():
    import torch
    return (torch.bfloat16, torch.int16) + ((torch.uint16,) if hasattr(torch, "uint16") else ())


def _op_args(W, x, g, out_name, out, out_dtypes, scratch=None, logits=None):
    """Types and shapes of every argument first, then the scratch size, then
    that all tensors share one CUDA device.  Returns (R, N, K, device)."""
    import torch
    _need(x, "x", (torch.float32,), cuda=False)
    if x.dim() != 2:
        raise ValueError(f"x: expected [R, K], got shape {tuple(x.shape)}")
    R, K = x.shape
    if not isinstance(W, torch.Tensor) or W.dim() != 2:
        raise ValueError("W: expected a [N, K] tensor")
    N = W.shape[0]
    _need(W, "W", _bf16_types(), (N, K), cuda=False)
    _need(g, "g", _bf16_types(), (K,), cuda=False)
    _need(out, out_name, out_dtypes, (R, N) if out_name == "y" else (R,), cuda=False)
    named = [("x", x), ("W", W), ("g", g), (out_name, out)]
    if logits is not None:
        _need(logits, "logits", (torch.float32,), (R, N), cuda=False)
        named.append(("logits", logits))
    if scratch is not None:
        _need(scratch, "scratch", (torch.uint8,), cuda=False)
        # the kernels write status words, counters and partials across the
        # whole documented scratch size; the C side cannot see the length
        need = int(ocrdec_op_scratch_bytes())
        if scratch.numel() < need:
            raise ValueError(f"scratch: {scratch.numel()} bytes, need at least {need} (op_scratch() allocates it)")
        named.append(("scratch", scratch))
    for name, t in named:
        if t.device != x.device:
            raise ValueError(f"{name}: on {t.device}, but x is on {x.device}; all tensors must share one device")
    for name, t in named:
        if not t.is_cuda:
            raise ValueError(f"{name}: must be a CUDA tensor")
    return R, N, K, x.device


def op_norm_gemv(W, x, g, eps, y, scratch, stream=None):
    import torch
    R, N, K, dev = _op_args(W, x, g, "y", y, (torch.float32,), scratch)
    with torch.cuda.device(dev):  # the kernel runs on the tensors' device
        check(ocrdec_op_norm_gemv(W.data_ptr(), x.data_ptr(), g.data_ptr(), eps, R, N, K, y.data_ptr(),
                                  scratch.data_ptr(), _stream(stream)), "ocrdec_op_norm_gemv")


def op_lm_argmax(W, x, g, eps, tok, logits, scratch, stream=None):
    import torch
    R, N, K, dev = _op_args(W, x, g, "tok", tok, (torch.int32,), scratch, logits)
    with torch.cuda.device(dev):
        check(ocrdec_op_lm_argmax(W.data_ptr(), x.data_ptr(), g.data_ptr(), eps, R, N, K, tok.data_ptr(),
                                  _ptr(logits), scratch.data_ptr(), _stream(stream)), "ocrdec_op_lm_argmax")


def op_lm_argmax_static(W, x, g, eps, tok, logits, stream=None):
    """op_lm_argmax on the library's fixed per-device scratch (allocates nothing)."""
    import torch
    R, N, K, dev = _op_args(W, x, g, "tok", tok, (torch.int32,), None, logits)
    with torch.cuda.device(dev):  # the scratch used is the one of this device
        check(ocrdec_op_lm_argmax_static(W.data_ptr(), x.data_ptr(), g.data_ptr(), eps, R, N, K, tok.data_ptr(),
                                         _ptr(logits), _stream(stream)), "ocrdec_op_lm_argmax_static")
