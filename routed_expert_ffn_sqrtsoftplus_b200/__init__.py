"""B200 (sm_100a) DeepSeek-V4.1-Flash routed-expert FFN layer with sqrtsoftplus routing.

A thin ctypes binding of the C ABI in include/moe.h. It only marshals torch
tensors into pointers and streams: every step of the layer runs in the CUDA
kernels of libmoe_b200.so. There is no CPU fallback; if the library is missing
or no CUDA device is present the calls raise.

    from routed_expert_ffn_sqrtsoftplus_b200 import MoELayer
    layer = MoELayer(hidden=5120, inter=2304, n_routed=384, n_shared=1, top_k=6,
                     max_tokens=32, router_w=wg, w1=w1, w3=w3, w2=w2,
                     sh_w1=s1, sh_w3=s3, sh_w2=s2)
    y = layer(x)                       # x, y: BF16 [T, 5120] on the GPU
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_OOM, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE = range(7)
MOE_DT_BF16, MOE_DT_MXFP4, MOE_DT_MXFP8 = 0, 1, 2

# moe_buffer ids
(BUF_LOGITS, BUF_TOPK_IDX, BUF_TOPK_W, BUF_COUNTS, BUF_OFFSETS, BUF_PERM, BUF_INV, BUF_H, BUF_XQ, BUF_XQ_SCALES,
 BUF_HQ, BUF_HQ_SCALES, BUF_NTILES, BUF_TILES_GU, BUF_TILES_DN) = range(15)

EXPORTED = ("moe_create", "moe_forward", "moe_forward_host", "moe_get_status", "moe_status_string",
            "moe_destroy", "moe_abi_version", "moe_quantize_mxfp4", "moe_inspect", "moe_set_wait_timeout",
            "moe_selftest_wait_timeout", "moe_get_info", "moe_profile_begin", "moe_profile_end",
            "moe_num_kernel_kinds", "moe_kernel_name", "moe_route_noalloc", "moe_quantize_mxfp8",
            "moe_set_hash_table", "moe_forward_hashed", "moe_fill_workspace", "moe_create_ep",
            "moe_forward_partial", "moe_read_bandwidth", "moe_forward_host_async", "moe_forward_host_wait")


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = _status_name(status)
        super().__init__(f"{what}: {name}" if what else name)


class _Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_routed", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("top_k", ctypes.c_int32), ("max_tokens", ctypes.c_int32),
                ("route_scale", ctypes.c_float), ("swiglu_limit", ctypes.c_float),
                ("expert_dtype", ctypes.c_int32)]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("router_w", "router_bias", "w1", "w3", "w2", "s1", "s3", "s2",
                                              "sh_w1", "sh_w3", "sh_w2")]


class _Info(ctypes.Structure):
    _fields_ = [("weight_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
                ("num_sms", ctypes.c_int32), ("last_tokens", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmoe_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m routed_expert_ffn_sqrtsoftplus_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, U64, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_int64
        sig = {
            "moe_create": (I32, [ctypes.POINTER(_Config), ctypes.POINTER(_Weights), P, ctypes.POINTER(P)]),
            "moe_forward": (I32, [P, P, I32, P, P, P, P]),
            "moe_forward_host": (I32, [P, P, I32, P, P, P, P]),
            "moe_forward_host_async": (I32, [P, P, I32, P, P]),
            "moe_forward_host_wait": (I32, [P, P]),
            "moe_get_status": (I32, [P]),
            "moe_status_string": (ctypes.c_char_p, [I32]),
            "moe_destroy": (None, [P]),
            "moe_abi_version": (I32, []),
            "moe_quantize_mxfp4": (I32, [P, I64, I32, P, P, P]),
            "moe_quantize_mxfp8": (I32, [P, I64, I32, P, P, P]),
            "moe_set_hash_table": (I32, [P, P, I32, P]),
            "moe_fill_workspace": (I32, [P, I32, P]),
            "moe_create_ep": (I32, [ctypes.POINTER(_Config), ctypes.POINTER(_Weights), I32, I32, P,
                                    ctypes.POINTER(P)]),
            "moe_forward_partial": (I32, [P, P, I32, P, P, P, P]),
            "moe_read_bandwidth": (I32, [P, ctypes.c_size_t, I32, P, ctypes.POINTER(ctypes.c_double)]),
            "moe_forward_hashed": (I32, [P, P, P, I32, P, P, P, P]),
            "moe_inspect": (I32, [P, I32, P, ctypes.c_size_t, P]),
            "moe_set_wait_timeout": (I32, [P, U64]),
            "moe_selftest_wait_timeout": (I32, [P, U64, P]),
            "moe_get_info": (I32, [P, ctypes.POINTER(_Info)]),
            "moe_profile_begin": (I32, [P, I32]),
            "moe_profile_end": (I32, [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I64), I32]),
            "moe_num_kernel_kinds": (I32, []),
            "moe_kernel_name": (ctypes.c_char_p, [I32]),
            "moe_route_noalloc": (I32, [P, P, P, I32, I32, I32, I32, ctypes.c_float, P, P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _status_name(s: int) -> str:
    try:
        return lib().moe_status_string(s).decode()
    except Exception:
        return f"status {s}"


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoEError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype, shape=None, device_type="cuda"):
    if t.device.type != device_type:
        raise ValueError(f"{name} must be on {device_type}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def kernel_names():
    L = lib()
    return [L.moe_kernel_name(i).decode() for i in range(L.moe_num_kernel_kinds())]


def quantize_mxfp4(w: torch.Tensor, stream=None):
    """BF16 [..., K] (CUDA) -> (packed E2M1 uint8 [..., K/2], E8M0 uint8 [..., K/32]) on the device."""
    _need(w, "w", torch.bfloat16)
    K = w.shape[-1]
    rows = w.numel() // K
    packed = torch.empty(w.shape[:-1] + (K // 2,), dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.shape[:-1] + (K // 32,), dtype=torch.uint8, device=w.device)
    _check(lib().moe_quantize_mxfp4(_ptr(w), rows, K, _ptr(packed), _ptr(scales), _stream(stream)),
           "moe_quantize_mxfp4")
    return packed, scales


def quantize_mxfp8(w: torch.Tensor, stream=None):
    """BF16 [..., K] (CUDA) -> (E4M3 codes uint8 [..., K], E8M0 uint8 [..., K/32]) on the device."""
    _need(w, "w", torch.bfloat16)
    K = w.shape[-1]
    rows = w.numel() // K
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.shape[:-1] + (K // 32,), dtype=torch.uint8, device=w.device)
    _check(lib().moe_quantize_mxfp8(_ptr(w), rows, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "moe_quantize_mxfp8")
    return codes, scales


def read_bandwidth(buf: torch.Tensor, reps: int = 5, stream=None) -> float:
    """Read-only streaming bandwidth (GB/s) of the device holding `buf` (a large CUDA tensor)."""
    if buf.device.type != "cuda" or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous CUDA tensor")
    g = ctypes.c_double(0.0)
    _check(lib().moe_read_bandwidth(_ptr(buf), buf.numel() * buf.element_size(), reps, _stream(stream),
                                    ctypes.byref(g)), "moe_read_bandwidth")
    return g.value


class MoELayer:
    """One routed-expert FFN layer resident on the current CUDA device."""

    def __init__(self, *, hidden: int, inter: int, n_routed: int, n_shared: int, top_k: int, max_tokens: int,
                 router_w: torch.Tensor, w1: torch.Tensor, w3: torch.Tensor, w2: torch.Tensor,
                 sh_w1: Optional[torch.Tensor] = None, sh_w3: Optional[torch.Tensor] = None,
                 sh_w2: Optional[torch.Tensor] = None, router_bias: Optional[torch.Tensor] = None,
                 s1: Optional[torch.Tensor] = None, s3: Optional[torch.Tensor] = None,
                 s2: Optional[torch.Tensor] = None, route_scale: float = 1.5, swiglu_limit: float = 10.0,
                 expert_dtype: str = "bf16", expert_begin: int = 0, expert_count: Optional[int] = None,
                 stream=None):
        """expert_begin / expert_count: hold only that window of the routed experts
        (expert parallelism; w1 / w3 / w2 and s1 / s3 / s2 then hold expert_count
        experts); such a layer computes partial outputs only (forward_partial)."""
        self._h = ctypes.c_void_p(None)
        L = lib()
        H, I, E, S = hidden, inter, n_routed, n_shared
        Ec = E if expert_count is None else expert_count
        _need(router_w, "router_w", torch.bfloat16, (E, H))
        if router_bias is not None:
            _need(router_bias, "router_bias", torch.float32, (E,))
        if expert_dtype == "bf16":
            _need(w1, "w1", torch.bfloat16, (Ec, I, H)); _need(w3, "w3", torch.bfloat16, (Ec, I, H))
            _need(w2, "w2", torch.bfloat16, (Ec, H, I))
            dt = MOE_DT_BF16
        elif expert_dtype in ("mxfp4", "mxfp8"):
            div = 2 if expert_dtype == "mxfp4" else 1
            _need(w1, "w1", torch.uint8, (Ec, I, H // div)); _need(w3, "w3", torch.uint8, (Ec, I, H // div))
            _need(w2, "w2", torch.uint8, (Ec, H, I // div))
            for n, t, shp in (("s1", s1, (Ec, I, H // 32)), ("s3", s3, (Ec, I, H // 32)),
                              ("s2", s2, (Ec, H, I // 32))):
                if t is None:
                    raise ValueError(f"{n} is required for {expert_dtype} experts")
                _need(t, n, torch.uint8, shp)
            dt = MOE_DT_MXFP4 if expert_dtype == "mxfp4" else MOE_DT_MXFP8
        else:
            raise ValueError("expert_dtype must be 'bf16', 'mxfp4' or 'mxfp8'")
        if S > 0:
            _need(sh_w1, "sh_w1", torch.bfloat16, (S, I, H)); _need(sh_w3, "sh_w3", torch.bfloat16, (S, I, H))
            _need(sh_w2, "sh_w2", torch.bfloat16, (S, H, I))
        self.cfg = _Config(H, I, E, S, top_k, max_tokens, float(route_scale), float(swiglu_limit), dt)
        wts = _Weights(_ptr(router_w), _ptr(router_bias), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(s1), _ptr(s3),
                       _ptr(s2), _ptr(sh_w1), _ptr(sh_w3), _ptr(sh_w2))
        st = _stream(stream)
        if expert_count is None and expert_begin == 0:
            _check(L.moe_create(ctypes.byref(self.cfg), ctypes.byref(wts), st, ctypes.byref(self._h)), "moe_create")
        else:
            _check(L.moe_create_ep(ctypes.byref(self.cfg), ctypes.byref(wts), expert_begin, Ec, st,
                                   ctypes.byref(self._h)), "moe_create_ep")
        self.expert_begin, self.expert_count = expert_begin, Ec
        # The library copied the weights on `st`; wait so the caller may free its tensors.
        torch.cuda.synchronize()
        self.hidden, self.inter, self.n_routed, self.n_shared, self.top_k = H, I, E, S, top_k
        self.max_tokens = max_tokens
        self.device = router_w.device

    # ------------------------------------------------------------------ forward
    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, topk_idx: Optional[torch.Tensor] = None,
                topk_w: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        _need(x, "x", torch.bfloat16, (T, self.hidden))
        if x.device != self.device:
            raise ValueError(f"x is on {x.device}, the layer on {self.device}")
        if out is None:
            out = torch.empty_like(x)
        _need(out, "out", torch.bfloat16, (T, self.hidden))
        if out.device != self.device:
            raise ValueError(f"out is on {out.device}, the layer on {self.device}")
        if topk_idx is not None:
            _need(topk_idx, "topk_idx", torch.int32, (T, self.top_k))
        if topk_w is not None:
            _need(topk_w, "topk_w", torch.float32, (T, self.top_k))
        _check(lib().moe_forward(self._h, _ptr(x), T, _ptr(out), _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
               "moe_forward")
        return out

    __call__ = forward

    def forward_partial(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """This layer's share of an expert-parallel layer, fp32 [T, H]: the selected
        slots whose expert lies in its window (plus the shared experts it holds)."""
        T = x.shape[0]
        _need(x, "x", torch.bfloat16, (T, self.hidden))
        if out is None:
            out = torch.empty((T, self.hidden), dtype=torch.float32, device=x.device)
        _need(out, "out", torch.float32, (T, self.hidden))
        for n, t in (("x", x), ("out", out)):
            if t.device != self.device:
                raise ValueError(f"{n} is on {t.device}, the layer on {self.device}")
        _check(lib().moe_forward_partial(self._h, _ptr(x), T, _ptr(out), None, None, _stream(stream)),
               "moe_forward_partial")
        return out

    def set_hash_table(self, table: torch.Tensor, stream=None):
        """Vocabulary table int32 [vocab, top_k] of a hash-routed layer (copied by the library)."""
        _need(table, "table", torch.int32)
        if table.dim() != 2 or table.shape[1] != self.top_k:
            raise ValueError(f"table must be [vocab, {self.top_k}]")
        _check(lib().moe_set_hash_table(self._h, _ptr(table), table.shape[0], _stream(stream)),
               "moe_set_hash_table")

    def forward_hashed(self, x: torch.Tensor, token_ids: torch.Tensor, out: Optional[torch.Tensor] = None,
                       topk_idx: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
        """The layer with hash routing: experts from the table row of each token's id."""
        T = x.shape[0]
        _need(x, "x", torch.bfloat16, (T, self.hidden))
        _need(token_ids, "token_ids", torch.int32, (T,))
        if out is None:
            out = torch.empty_like(x)
        _need(out, "out", torch.bfloat16, (T, self.hidden))
        for n, t in (("x", x), ("token_ids", token_ids), ("out", out)):
            if t.device != self.device:
                raise ValueError(f"{n} is on {t.device}, the layer on {self.device}")
        if topk_idx is not None:
            _need(topk_idx, "topk_idx", torch.int32, (T, self.top_k))
        if topk_w is not None:
            _need(topk_w, "topk_w", torch.float32, (T, self.top_k))
        _check(lib().moe_forward_hashed(self._h, _ptr(x), _ptr(token_ids), T, _ptr(out), _ptr(topk_idx),
                                        _ptr(topk_w), _stream(stream)), "moe_forward_hashed")
        return out

    def forward_with_routing(self, x: torch.Tensor, stream=None):
        T = x.shape[0]
        idx = torch.empty((T, self.top_k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.top_k), dtype=torch.float32, device=x.device)
        y = self.forward(x, topk_idx=idx, topk_w=w, stream=stream)
        return y, idx, w

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, topk_idx_host: Optional[torch.Tensor] = None,
                     topk_w_host: Optional[torch.Tensor] = None, stream=None):
        """Host buffers in, host buffers out (copies enqueued on the stream; sync before reading)."""
        T = x_host.shape[0]
        _need(x_host, "x_host", torch.bfloat16, (T, self.hidden), "cpu")
        _need(y_host, "y_host", torch.bfloat16, (T, self.hidden), "cpu")
        if topk_idx_host is not None:
            _need(topk_idx_host, "topk_idx_host", torch.int32, (T, self.top_k), "cpu")
        if topk_w_host is not None:
            _need(topk_w_host, "topk_w_host", torch.float32, (T, self.top_k), "cpu")
        _check(lib().moe_forward_host(self._h, _ptr(x_host), T, _ptr(y_host), _ptr(topk_idx_host),
                                      _ptr(topk_w_host), _stream(stream)), "moe_forward_host")

    def forward_host_async(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None):
        """Pipelined host buffers in and out: the copies run on the library's own streams
        and overlap the neighbouring calls' layers. Call forward_host_wait(stream) and
        synchronise the stream before reading y_host or reusing a call's buffers."""
        T = x_host.shape[0]
        _need(x_host, "x_host", torch.bfloat16, (T, self.hidden), "cpu")
        _need(y_host, "y_host", torch.bfloat16, (T, self.hidden), "cpu")
        _check(lib().moe_forward_host_async(self._h, _ptr(x_host), T, _ptr(y_host), _stream(stream)),
               "moe_forward_host_async")

    def forward_host_wait(self, stream=None):
        """Make the stream wait for every copy-out of forward_host_async so far."""
        _check(lib().moe_forward_host_wait(self._h, _stream(stream)), "moe_forward_host_wait")

    # ------------------------------------------------------------------ inspection
    def inspect(self, what: int, out: torch.Tensor, stream=None) -> torch.Tensor:
        nbytes = out.numel() * out.element_size()
        _check(lib().moe_inspect(self._h, what, _ptr(out), nbytes, _stream(stream)), "moe_inspect")
        return out

    def fill_workspace(self, byte_value: int, stream=None):
        """Overwrite every per-forward scratch buffer with one byte value (a debugging aid)."""
        _check(lib().moe_fill_workspace(self._h, int(byte_value), _stream(stream)), "moe_fill_workspace")

    def status(self) -> int:
        return lib().moe_get_status(self._h)

    def info(self) -> dict:
        i = _Info()
        _check(lib().moe_get_info(self._h, ctypes.byref(i)), "moe_get_info")
        return dict(weight_bytes=i.weight_bytes, workspace_bytes=i.workspace_bytes, num_sms=i.num_sms,
                    last_tokens=i.last_tokens)

    def set_wait_timeout(self, ns: int):
        _check(lib().moe_set_wait_timeout(self._h, int(ns)), "moe_set_wait_timeout")

    def selftest_wait_timeout(self, ns: int, stream=None):
        _check(lib().moe_selftest_wait_timeout(self._h, int(ns), _stream(stream)), "moe_selftest_wait_timeout")

    def profile_begin(self, max_calls: int):
        _check(lib().moe_profile_begin(self._h, max_calls), "moe_profile_begin")

    def profile_end(self) -> dict:
        L = lib()
        n = L.moe_num_kernel_kinds()
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int64 * n)()
        _check(L.moe_profile_end(self._h, ms, cnt, n), "moe_profile_end")
        return {kernel_names()[i]: (ms[i], cnt[i]) for i in range(n) if cnt[i] > 0}

    def close(self):
        if self._h:
            lib().moe_destroy(self._h)
            self._h = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @classmethod
    def from_layer(cls, layer: dict, *, top_k: int, max_tokens: int, route_scale: float = 1.5,
                   swiglu_limit: float = 10.0, mx: Optional[dict] = None, expert_window=None,
                   with_shared: bool = True, stream=None) -> "MoELayer":
        """Build from a dict of tensors (x ignored): wg, bias, w1, w3, w2, sh_w1, sh_w3, sh_w2.

        With ``mx`` = dict(w1, s1, w3, s3, w2, s2) of MXFP4 (packed, w1 [E, I, H/2]) or
        MXFP8 (w1 [E, I, H]) tensors the routed experts are stored in that format.
        """
        E, I, H = layer["w1"].shape
        S = layer["sh_w1"].shape[0] if (with_shared and layer.get("sh_w1") is not None) else 0
        sh = {n: (layer.get(n) if S > 0 else None) for n in ("sh_w1", "sh_w3", "sh_w2")}
        b, c = (0, None) if expert_window is None else expert_window
        if expert_window is not None and not (0 <= b and 1 <= c and b + c <= E):
            raise ValueError(f"expert window {expert_window} is not inside [0, {E})")
        cut = (lambda t: t) if expert_window is None else (lambda t: t[b:b + c].contiguous())
        kw = dict(hidden=H, inter=I, n_routed=E, n_shared=S, top_k=top_k, max_tokens=max_tokens,
                  router_w=layer["wg"], router_bias=layer.get("bias"), route_scale=route_scale,
                  swiglu_limit=swiglu_limit, expert_begin=b, expert_count=c, stream=stream, **sh)
        if mx is None:
            return cls(w1=cut(layer["w1"]), w3=cut(layer["w3"]), w2=cut(layer["w2"]), expert_dtype="bf16", **kw)
        fmt = "mxfp8" if mx["w1"].shape[-1] == H else "mxfp4"
        return cls(w1=cut(mx["w1"]), w3=cut(mx["w3"]), w2=cut(mx["w2"]), s1=cut(mx["s1"]), s3=cut(mx["s3"]),
                   s2=cut(mx["s2"]), expert_dtype=fmt, **kw)
