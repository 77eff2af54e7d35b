"""Python binding of libling_moe.so, the B200 W4 g32 MoE-layer library.

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  The functions below carry the C ABI's names and arguments
(pointers are integers, streams are raw cudaStream_t values); `MoELayer`
wraps them for torch tensors.  The library must have been built
(`python -m weight_only_int4_fp32_b200.build`); the first call into it
raises if it is missing -- there is nothing else to fall back to.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "LING_MOE_OK", "LING_MOE_ERR_INVALID_ARG", "LING_MOE_ERR_CUDA", "LING_MOE_ERR_OOM",
    "LING_MOE_ERR_UNSUPPORTED", "LING_MOE_ERR_DEVICE_TIMEOUT", "LingMoEError",
    "ling_moe_config_t", "ling_moe_weights_t", "library_path", "load_library",
    "ling_moe_create", "ling_moe_create_mxfp4", "ling_moe_forward", "ling_moe_forward_ex", "ling_moe_forward_host",
    "ling_moe_status", "ling_moe_describe", "ling_moe_launch_count", "ling_moe_last_error",
    "ling_moe_destroy", "ling_moe_test_set_wait", "ling_moe_route_noalloc", "ling_moe_route_noalloc_status",
    "ling_moe_route_noalloc_test_set_wait", "ling_moe_set_kernel_timing",
    "ling_moe_kernel_times", "ling_moe_ep_t", "ling_moe_create_ep", "ling_moe_forward_partial",
    "ling_moe_round_bf16", "LING_MOE_FORMAT_INT4", "LING_MOE_FORMAT_MXFP4", "round_bf16",
    "MoELayer", "LMHeadFP8", "EXPORTED",
]

LING_MOE_OK = 0
LING_MOE_ERR_INVALID_ARG = -1
LING_MOE_ERR_CUDA = -2
LING_MOE_ERR_OOM = -3
LING_MOE_ERR_UNSUPPORTED = -4
LING_MOE_ERR_DEVICE_TIMEOUT = -5
LING_MOE_FORMAT_INT4 = 0
LING_MOE_FORMAT_MXFP4 = 1

# every symbol include/ling_moe.h declares
EXPORTED = (
    "ling_moe_create", "ling_moe_create_mxfp4", "ling_moe_forward", "ling_moe_forward_ex",
    "ling_moe_forward_host", "ling_moe_status", "ling_moe_describe", "ling_moe_launch_count",
    "ling_moe_last_error", "ling_moe_destroy", "ling_moe_test_set_wait", "ling_moe_route_noalloc",
    "ling_moe_route_noalloc_status", "ling_moe_route_noalloc_test_set_wait", "ling_moe_set_kernel_timing",
    "ling_moe_kernel_times", "ling_moe_kernel_name", "ling_moe_create_ep", "ling_moe_forward_partial",
    "ling_moe_round_bf16",
    "ling_moe_lmhead_create", "ling_moe_lmhead_forward", "ling_moe_lmhead_forward_ex",
    "ling_moe_lmhead_forward_host", "ling_moe_lmhead_weights", "ling_moe_lmhead_status",
    "ling_moe_lmhead_launch_count", "ling_moe_lmhead_destroy", "ling_moe_lmhead_test_set_wait",
)

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.environ.get("LING_MOE_LIB", os.path.join(_HERE, "libling_moe.so"))


class LingMoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"ling_moe error {code}: {msg}")
        self.code = code


class ling_moe_config_t(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("num_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("group_size", ctypes.c_int), ("max_tokens", ctypes.c_int)]


class ling_moe_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_w", "router_bias", "gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s",
        "sh_gate", "sh_up", "sh_down")]


class ling_moe_ep_t(ctypes.Structure):
    _fields_ = [("expert_begin", ctypes.c_int), ("expert_count", ctypes.c_int), ("with_shared", ctypes.c_int),
                ("format", ctypes.c_int)]


_LIB = None


def load_library():
    """Load libling_moe.so once (raises ImportError if it is missing or stale)."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def _load():
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(
            f"libling_moe.so not found at {path}: build it with "
            "`python -m weight_only_int4_fp32_b200.build` (there is no fallback path)")
    L = ctypes.CDLL(path)
    vp, ci, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    sig = {
        "ling_moe_create": (ci, [ctypes.POINTER(ling_moe_config_t), ctypes.POINTER(ling_moe_weights_t),
                                 ctypes.POINTER(vp)]),
        "ling_moe_create_mxfp4": (ci, [ctypes.POINTER(ling_moe_config_t), ctypes.POINTER(ling_moe_weights_t),
                                       ctypes.POINTER(vp)]),
        "ling_moe_create_ep": (ci, [ctypes.POINTER(ling_moe_config_t), ctypes.POINTER(ling_moe_weights_t),
                                    ctypes.POINTER(ling_moe_ep_t), ctypes.POINTER(vp)]),
        "ling_moe_forward_partial": (ci, [vp, vp, ci, vp, vp, vp, vp]),
        "ling_moe_round_bf16": (ci, [vp, vp, ctypes.c_size_t, vp]),
        "ling_moe_forward": (ci, [vp, vp, ci, vp, vp]),
        "ling_moe_forward_ex": (ci, [vp, vp, ci, vp, vp, vp, vp]),
        "ling_moe_forward_host": (ci, [vp, vp, ci, vp, vp]),
        "ling_moe_status": (ci, [vp, vp]),
        "ling_moe_describe": (ctypes.c_char_p, [vp]),
        "ling_moe_launch_count": (i64, [vp]),
        "ling_moe_last_error": (ctypes.c_char_p, []),
        "ling_moe_destroy": (None, [vp]),
        "ling_moe_test_set_wait": (ci, [vp, ci, ctypes.c_uint64]),
        "ling_moe_route_noalloc": (ci, [vp, ci, vp, vp, ci, ci, vp, vp, vp]),
        "ling_moe_route_noalloc_status": (ci, [vp]),
        "ling_moe_route_noalloc_test_set_wait": (ci, [ci, ctypes.c_uint64]),
        "ling_moe_set_kernel_timing": (ci, [vp, ci]),
        "ling_moe_kernel_times": (ci, [vp, ctypes.POINTER(ctypes.c_float), ci, ctypes.POINTER(ci)]),
        "ling_moe_kernel_name": (ctypes.c_char_p, [vp, ci]),
        "ling_moe_lmhead_create": (ci, [vp, ci, ci, ctypes.POINTER(vp)]),
        "ling_moe_lmhead_forward": (ci, [vp, vp, ci, vp, vp]),
        "ling_moe_lmhead_forward_ex": (ci, [vp, vp, ci, vp, vp, vp, vp]),
        "ling_moe_lmhead_forward_host": (ci, [vp, vp, ci, vp, vp]),
        "ling_moe_lmhead_weights": (ci, [vp, vp, vp, vp]),
        "ling_moe_lmhead_status": (ci, [vp, vp]),
        "ling_moe_lmhead_launch_count": (i64, [vp]),
        "ling_moe_lmhead_destroy": (None, [vp]),
        "ling_moe_lmhead_test_set_wait": (ci, [vp, ci, ctypes.c_uint64]),
    }
    for name, (res, args) in sig.items():
        try:
            f = getattr(L, name)
        except AttributeError as e:
            raise ImportError(f"{path} lacks {name}: rebuild it "
                              "(`python -m weight_only_int4_fp32_b200.build`)") from e
        f.restype = res
        f.argtypes = args
    return L


class _LazyLib:
    def __getattr__(self, name):
        return getattr(load_library(), name)


lib = _LazyLib()


def ling_moe_last_error() -> str:
    return lib.ling_moe_last_error().decode()


def _check(rc: int) -> int:
    if rc != LING_MOE_OK:
        raise LingMoEError(rc, ling_moe_last_error())
    return rc


def ling_moe_create(cfg: ling_moe_config_t, weights: ling_moe_weights_t) -> int:
    h = ctypes.c_void_p()
    _check(lib.ling_moe_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(h)))
    return h.value


def ling_moe_create_mxfp4(cfg: ling_moe_config_t, weights: ling_moe_weights_t) -> int:
    h = ctypes.c_void_p()
    _check(lib.ling_moe_create_mxfp4(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(h)))
    return h.value


def ling_moe_create_ep(cfg: ling_moe_config_t, weights: ling_moe_weights_t, ep: ling_moe_ep_t) -> int:
    h = ctypes.c_void_p()
    _check(lib.ling_moe_create_ep(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(ep), ctypes.byref(h)))
    return h.value


def ling_moe_forward_partial(h: int, x: int, T: int, partial: int, topk_idx: int = None, topk_w: int = None,
                             stream: int = 0) -> int:
    return _check(lib.ling_moe_forward_partial(h, x, T, partial, topk_idx, topk_w, stream))


def ling_moe_round_bf16(inp: int, out: int, n: int, stream: int = 0) -> int:
    return _check(lib.ling_moe_round_bf16(inp, out, n, stream))


def ling_moe_set_kernel_timing(h: int, on: bool) -> int:
    return _check(lib.ling_moe_set_kernel_timing(h, 1 if on else 0))


def ling_moe_kernel_times(h: int) -> list:
    """[(kernel name, ms)] of the last forward call issued with timing on."""
    ms = (ctypes.c_float * 16)()
    n = ctypes.c_int(0)
    _check(lib.ling_moe_kernel_times(h, ms, 16, ctypes.byref(n)))
    return [(lib.ling_moe_kernel_name(h, i).decode(), float(ms[i])) for i in range(n.value)]


def ling_moe_forward(h: int, x: int, T: int, out: int, stream: int = 0) -> int:
    return _check(lib.ling_moe_forward(h, x, T, out, stream))


def ling_moe_forward_ex(h: int, x: int, T: int, out: int, topk_idx: int, topk_w: int,
                        stream: int = 0) -> int:
    return _check(lib.ling_moe_forward_ex(h, x, T, out, topk_idx, topk_w, stream))


def ling_moe_forward_host(h: int, x_host: int, T: int, out_host: int, stream: int = 0) -> int:
    return _check(lib.ling_moe_forward_host(h, x_host, T, out_host, stream))


def ling_moe_status(h: int, stream: int = 0) -> int:
    """Returns the status code (does not raise on DEVICE_TIMEOUT)."""
    return lib.ling_moe_status(h, stream)


def ling_moe_describe(h: int) -> str:
    return lib.ling_moe_describe(h).decode()


def ling_moe_launch_count(h: int) -> int:
    return lib.ling_moe_launch_count(h)


def ling_moe_destroy(h: int) -> None:
    lib.ling_moe_destroy(h)


def ling_moe_test_set_wait(h: int, skip_arrive_cta: int, wait_limit_ns: int) -> int:
    return _check(lib.ling_moe_test_set_wait(h, skip_arrive_cta, wait_limit_ns))


def ling_moe_route_noalloc(x: int, T: int, router_w: int, router_bias, num_experts: int, top_k: int,
                           topk_idx: int, topk_w: int, stream: int = 0) -> int:
    """Routing with the library's static scratch; allocates nothing (see ling_moe.h)."""
    return _check(lib.ling_moe_route_noalloc(x, T, router_w, router_bias or None, num_experts, top_k,
                                             topk_idx, topk_w, stream))


def ling_moe_route_noalloc_status(stream: int = 0) -> int:
    """LING_MOE_OK, or LING_MOE_ERR_DEVICE_TIMEOUT if a routing wait gave up since the last check
    (returned, not raised, like MoELayer.status)."""
    rc = lib.ling_moe_route_noalloc_status(stream)
    if rc not in (LING_MOE_OK, LING_MOE_ERR_DEVICE_TIMEOUT):
        raise LingMoEError(rc, ling_moe_last_error())
    return rc


def ling_moe_route_noalloc_test_set_wait(skip_cta: int, wait_limit_ns: int) -> int:
    return _check(lib.ling_moe_route_noalloc_test_set_wait(skip_cta, wait_limit_ns))


def _require(t, shape, dtype, cuda: bool, name: str):
    """Raise ValueError unless t is a contiguous tensor of this shape and dtype
    on the GPU (cuda) or the host; the C calls trust the sizes they are given."""
    if (tuple(t.shape) != tuple(shape) or t.dtype != dtype or bool(t.is_cuda) != cuda
            or not t.is_contiguous()):
        where = "CUDA" if cuda else "host"
        raise ValueError(f"{name} must be a contiguous {where} {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def round_bf16(partial, out=None, stream=None):
    """bf16 round-to-nearest-even of an fp32 CUDA tensor (ling_moe_round_bf16):
    the last step of an expert-parallel combine."""
    import torch
    if not partial.is_cuda or partial.dtype != torch.float32 or not partial.is_contiguous():
        raise ValueError("partial must be a contiguous CUDA float32 tensor")
    if out is None:
        out = torch.empty(partial.shape, dtype=torch.bfloat16, device=partial.device)
    _require(out, tuple(partial.shape), torch.bfloat16, True, "out")
    s = torch.cuda.current_stream().cuda_stream if stream is None else getattr(stream, "cuda_stream", stream)
    ling_moe_round_bf16(partial.data_ptr(), out.data_ptr(), partial.numel(), s)
    return out


class MoELayer:
    """One MoE layer on the current CUDA device, built from torch tensors.

    `weights` maps the canonical names (router_w, router_bias, gate_q, gate_s,
    up_q, up_s, down_q, down_s, sh_gate, sh_up, sh_down) to contiguous CUDA
    tensors; they are copied, so they may be freed after construction.
    fmt="int4" (W4 g32, bf16 scales) or "mxfp4" (E2M1 codes, E8M0 scale bytes).
    """

    def __init__(self, weights: dict, top_k: int = 8, max_tokens: int = 1, group_size: int = 32,
                 fmt: str = "int4", ep: tuple | None = None):
        """ep = (expert_begin, expert_count, with_shared): an expert-parallel
        handle (ling_moe_create_ep) whose routed weights hold only experts
        [expert_begin, expert_begin + expert_count) of the router's E; it
        serves forward_partial only."""
        import torch  # device memory and streams only
        rw = weights["router_w"]
        E, H = rw.shape
        I = (weights["sh_gate"] if weights.get("sh_gate") is not None else weights["gate_q"][0]).shape[0]
        for k, v in weights.items():
            if v is not None and (not v.is_cuda or not v.is_contiguous()):
                raise ValueError(f"{k} must be a contiguous CUDA tensor")
        cfg = ling_moe_config_t(H, I, E, top_k, group_size, max_tokens)
        ptr = lambda n: (weights[n].data_ptr() if weights.get(n) is not None else None)
        w = ling_moe_weights_t(*(ptr(n) for n, _ in ling_moe_weights_t._fields_))
        self.E, self.H, self.I, self.k, self.max_tokens = E, H, I, top_k, max_tokens
        if fmt not in ("int4", "mxfp4"):
            raise ValueError("fmt must be 'int4' or 'mxfp4'")
        self.ep = ep
        if ep is not None:
            b, n, sh = ep
            spec = ling_moe_ep_t(int(b), int(n), int(bool(sh)),
                                 LING_MOE_FORMAT_MXFP4 if fmt == "mxfp4" else LING_MOE_FORMAT_INT4)
            self.handle = ling_moe_create_ep(cfg, w, spec)
        else:
            self.handle = (ling_moe_create_mxfp4 if fmt == "mxfp4" else ling_moe_create)(cfg, w)
        self._torch = torch

    def _stream(self, stream):
        if stream is None:
            return self._torch.cuda.current_stream().cuda_stream
        return getattr(stream, "cuda_stream", stream)

    def forward(self, x, out=None, stream=None, return_routing: bool = False):
        torch = self._torch
        if x.dim() != 2:
            raise ValueError("x must be 2-D [T, hidden]")
        T = x.shape[0]
        _require(x, (T, self.H), torch.bfloat16, True, "x")
        if out is None:
            out = torch.empty_like(x)
        _require(out, (T, self.H), torch.bfloat16, True, "out")
        s = self._stream(stream)
        if return_routing:
            idx = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
            w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
            ling_moe_forward_ex(self.handle, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(),
                                w.data_ptr(), s)
            return out, idx, w
        ling_moe_forward(self.handle, x.data_ptr(), T, out.data_ptr(), s)
        return out

    __call__ = forward

    def forward_partial(self, x, out=None, stream=None, return_routing: bool = False):
        """fp32 [T, hidden]: the sum of the terms this handle computes (all of
        the layer on an ordinary handle), before the bf16 rounding."""
        torch = self._torch
        if x.dim() != 2:
            raise ValueError("x must be 2-D [T, hidden]")
        T = x.shape[0]
        _require(x, (T, self.H), torch.bfloat16, True, "x")
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.float32, device=x.device)
        _require(out, (T, self.H), torch.float32, True, "out")
        s = self._stream(stream)
        idx = w = None
        if return_routing:
            idx = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
            w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        ling_moe_forward_partial(self.handle, x.data_ptr(), T, out.data_ptr(),
                                 idx.data_ptr() if idx is not None else None,
                                 w.data_ptr() if w is not None else None, s)
        return (out, idx, w) if return_routing else out

    def forward_host(self, x_host, out_host=None, stream=None):
        torch = self._torch
        T = x_host.shape[0]
        _require(x_host, (T, self.H), torch.bfloat16, False, "x_host")
        if out_host is None:
            out_host = torch.empty_like(x_host)
        _require(out_host, (T, self.H), torch.bfloat16, False, "out_host")
        ling_moe_forward_host(self.handle, x_host.data_ptr(), T, out_host.data_ptr(), self._stream(stream))
        return out_host

    def status(self, stream=None) -> int:
        return ling_moe_status(self.handle, self._stream(stream))

    def describe(self) -> str:
        return ling_moe_describe(self.handle)

    def launch_count(self) -> int:
        return ling_moe_launch_count(self.handle)

    def set_kernel_timing(self, on: bool = True):
        ling_moe_set_kernel_timing(self.handle, on)

    def kernel_times(self) -> list:
        """[(kernel name, ms)] of the last forward call issued with timing on."""
        return ling_moe_kernel_times(self.handle)

    def close(self):
        if getattr(self, "handle", None):
            ling_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class LMHeadFP8:
    """The online-FP8 LM head on the current CUDA device.

    `w` is the bf16 head [vocab, hidden] (contiguous CUDA tensor); it is
    quantised to e4m3 with one fp32 scale per row when the object is built
    and may be freed afterwards.  Each call quantises its tokens the same
    way and returns fp32 logits [T, vocab] (T <= 8).
    """

    MAX_TOKENS = 8

    def __init__(self, w):
        import torch  # device memory and streams only
        if w.dtype != torch.bfloat16 or not w.is_cuda or not w.is_contiguous() or w.dim() != 2:
            raise ValueError("w must be a contiguous 2-D bf16 CUDA tensor")
        self.vocab, self.hidden = w.shape
        h = ctypes.c_void_p()
        _check(lib.ling_moe_lmhead_create(w.data_ptr(), self.vocab, self.hidden, ctypes.byref(h)))
        self.handle = h.value
        self._torch = torch

    def _stream(self, stream):
        if stream is None:
            return self._torch.cuda.current_stream().cuda_stream
        return getattr(stream, "cuda_stream", stream)

    def forward(self, x, logits=None, stream=None, return_codes: bool = False):
        torch = self._torch
        if x.dim() != 2:
            raise ValueError("x must be 2-D [T, hidden]")
        T = x.shape[0]
        _require(x, (T, self.hidden), torch.bfloat16, True, "x")
        if logits is None:
            logits = torch.empty((T, self.vocab), dtype=torch.float32, device=x.device)
        _require(logits, (T, self.vocab), torch.float32, True, "logits")
        s = self._stream(stream)
        if return_codes:
            xq = torch.empty((T, self.hidden), dtype=torch.uint8, device=x.device)
            xs = torch.empty((T,), dtype=torch.float32, device=x.device)
            _check(lib.ling_moe_lmhead_forward_ex(self.handle, x.data_ptr(), T, logits.data_ptr(),
                                                  xq.data_ptr(), xs.data_ptr(), s))
            return logits, xq, xs
        _check(lib.ling_moe_lmhead_forward(self.handle, x.data_ptr(), T, logits.data_ptr(), s))
        return logits

    __call__ = forward

    def forward_host(self, x_host, logits_host=None, stream=None):
        torch = self._torch
        T = x_host.shape[0]
        _require(x_host, (T, self.hidden), torch.bfloat16, False, "x_host")
        if logits_host is None:
            logits_host = torch.empty((T, self.vocab), dtype=torch.float32, pin_memory=True)
        _require(logits_host, (T, self.vocab), torch.float32, False, "logits_host")
        _check(lib.ling_moe_lmhead_forward_host(self.handle, x_host.data_ptr(), T, logits_host.data_ptr(),
                                                self._stream(stream)))
        return logits_host

    def weights(self, stream=None):
        """(codes uint8 [vocab, hidden], scales fp32 [vocab]): the handle's quantised head, row-major."""
        torch = self._torch
        codes = torch.empty((self.vocab, self.hidden), dtype=torch.uint8, device="cuda")
        scales = torch.empty((self.vocab,), dtype=torch.float32, device="cuda")
        _check(lib.ling_moe_lmhead_weights(self.handle, codes.data_ptr(), scales.data_ptr(), self._stream(stream)))
        return codes, scales

    def status(self, stream=None) -> int:
        """Status code of the handle's device work (does not raise on DEVICE_TIMEOUT)."""
        return lib.ling_moe_lmhead_status(self.handle, self._stream(stream))

    def launch_count(self) -> int:
        return lib.ling_moe_lmhead_launch_count(self.handle)

    def test_set_wait(self, skip_cta: int, wait_limit_ns: int = 0):
        """Test hook (see ling_moe_lmhead_test_set_wait)."""
        _check(lib.ling_moe_lmhead_test_set_wait(self.handle, skip_cta, wait_limit_ns))

    def close(self):
        if getattr(self, "handle", None):
            lib.ling_moe_lmhead_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
