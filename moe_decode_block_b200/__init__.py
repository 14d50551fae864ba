"""MoE decode block for B200 (sm_100a): thin Python binding of the C ABI.

Every step of the forward runs in the CUDA kernels of ``libmoe_decode.so``;
this module only marshals arguments (PyTorch supplies device memory and
streams).  There is no CPU or PyTorch fallback: if the library is missing the
binding raises.

    blk = MoEDecode(hidden=7168, n_experts=384, top_k=8, inter=2048,
                    shared_inter=2048, max_batch=64)
    blk.forward(x, router_w, w13, w2, shared_w13, shared_w2, out, topk_ids, topk_w)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Union

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_decode.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_NO_DEVICE = -3
MOE_ERR_ARCH = -4
MOE_ERR_CUDA = -5
MOE_ERR_OUT_OF_MEMORY = -6
MOE_ERR_DEVICE_TIMEOUT = -7
MOE_ERR_DEVICE_PLAN = -8

# Entry points declared in include/moe_decode.h (checked by the tests).
EXPORTED = (
    "moe_decode_init", "moe_decode_forward", "moe_decode_forward_host",
    "moe_decode_forward_fp8",
    "moe_decode_destroy",
    "moe_decode_get_status", "moe_decode_get_stats", "moe_decode_error_string",
    "moe_decode_last_cuda_error", "moe_decode_last_cuda_error_string", "moe_decode_workspace_bytes",
    "moe_decode_set_timing_events", "moe_decode_set_wait_limit", "moe_router_topk_noalloc",
    "moe_router_topk_noalloc_status", "moe_decode_reduce_residual",
)
MOE_TIMING_EVENTS = 6
MOE_FLAG_TWO_STREAM = 1
MOE_FLAG_TCGEN05 = 2
MOE_FLAG_TEST_HOLD_PANEL = 4
MOE_FLAG_FP8_WEIGHTS = 8
MOE_FLAG_PARTIAL_SUM = 16
MOE_REDUCE_MAX_PARTS = 16


class Shapes(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32), ("n_shared", ctypes.c_int32),
        ("max_batch", ctypes.c_int32), ("router_bias", ctypes.c_void_p), ("flags", ctypes.c_uint32),
    ]


class Stats(ctypes.Structure):
    _fields_ = [
        ("forwards", ctypes.c_uint64), ("kernels_launched", ctypes.c_uint64),
        ("last_kernels", ctypes.c_int32), ("last_token_tiles", ctypes.c_int32),
        ("stages_up", ctypes.c_uint64 * 3), ("stages_down", ctypes.c_uint64 * 3),
    ]


class MoEDecodeError(RuntimeError):
    def __init__(self, code: int, what: str):
        lib = load_library()
        msg = lib.moe_decode_error_string(code).decode()
        if code == MOE_ERR_CUDA:
            msg += f" ({lib.moe_decode_last_cuda_error_string().decode()})"
        super().__init__(f"{what}: {msg} [{code}]")
        self.code = code


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libmoe_decode.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m moe_decode_block_b200.build` "
            "(the MoE decode block has no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.moe_decode_init.argtypes = [ctypes.POINTER(Shapes), ctypes.POINTER(ctypes.c_void_p)]
    lib.moe_decode_init.restype = I
    fwd = [P, P, P, P, P, P, P, P, P, P, ctypes.c_int32, P, P]
    lib.moe_decode_forward.argtypes = fwd
    lib.moe_decode_forward.restype = I
    lib.moe_decode_forward_host.argtypes = fwd
    lib.moe_decode_forward_host.restype = I
    lib.moe_decode_forward_fp8.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_int32, P, P]
    lib.moe_decode_forward_fp8.restype = I
    lib.moe_decode_destroy.argtypes = [P]
    lib.moe_decode_destroy.restype = I
    lib.moe_decode_get_status.argtypes = [P]
    lib.moe_decode_get_status.restype = I
    lib.moe_decode_get_stats.argtypes = [P, ctypes.POINTER(Stats)]
    lib.moe_decode_get_stats.restype = I
    lib.moe_decode_error_string.argtypes = [I]
    lib.moe_decode_error_string.restype = ctypes.c_char_p
    lib.moe_decode_last_cuda_error.argtypes = []
    lib.moe_decode_last_cuda_error.restype = I
    lib.moe_decode_last_cuda_error_string.argtypes = []
    lib.moe_decode_last_cuda_error_string.restype = ctypes.c_char_p
    lib.moe_decode_set_timing_events.argtypes = [P, P, ctypes.c_int32]
    lib.moe_decode_set_timing_events.restype = I
    lib.moe_router_topk_noalloc.argtypes = [P, P, P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_int32, P]
    lib.moe_router_topk_noalloc.restype = I
    lib.moe_router_topk_noalloc_status.argtypes = [P]
    lib.moe_router_topk_noalloc_status.restype = I
    lib.moe_decode_reduce_residual.argtypes = [P, ctypes.c_int32, P, P, ctypes.c_int32, ctypes.c_int32, P]
    lib.moe_decode_reduce_residual.restype = I
    lib.moe_decode_set_wait_limit.argtypes = [P, ctypes.c_uint32]
    lib.moe_decode_set_wait_limit.restype = I
    lib.moe_decode_workspace_bytes.argtypes = [ctypes.POINTER(Shapes)]
    lib.moe_decode_workspace_bytes.restype = ctypes.c_uint64
    _lib = lib
    return lib


def _check(code: int, what: str):
    if code != MOE_OK:
        raise MoEDecodeError(code, what)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_handle(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def router_topk_noalloc(x, router_w, topk_ids, topk_w, top_k: int, router_bias=None, stream=None):
    """Router scores, softmax, top-k and renormalised weights without a handle
    and without any device allocation (moe_router_topk_noalloc).  Make the
    first call on a device outside stream capture; calls that may overlap on
    the GPU share one scratch array and race."""
    import torch
    lib = load_library()
    sm = _stream_handle(stream if stream is not None else torch.cuda.current_stream())
    rc = lib.moe_router_topk_noalloc(_ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(topk_ids), _ptr(topk_w),
                                     int(x.shape[0]), int(router_w.shape[0]), int(router_w.shape[1]), int(top_k),
                                     sm)
    _check(rc, "moe_router_topk_noalloc")


def router_topk_noalloc_status(stream=None) -> int:
    """Synchronise `stream` and return the device status of the last
    allocation-free router call on the current device (MOE_OK or an
    MOE_ERR_* code); the status word is cleared."""
    import torch
    lib = load_library()
    sm = _stream_handle(stream if stream is not None else torch.cuda.current_stream())
    return lib.moe_router_topk_noalloc_status(sm)


def reduce_residual(partials, x, out, stream=None):
    """out = bf16(x + sum of the fp32 [B, H] partial sums in `partials`, in
    list order) -- moe_decode_reduce_residual; the tensors (or raw device
    pointers, e.g. a peer's mapped buffer) must be 16-byte aligned."""
    import torch
    lib = load_library()
    ptrs = (ctypes.c_void_p * len(partials))(*[_ptr(p) if hasattr(p, "data_ptr") else int(p) for p in partials])
    sm = _stream_handle(stream if stream is not None else torch.cuda.current_stream())
    rc = lib.moe_decode_reduce_residual(ptrs, len(partials), _ptr(x), _ptr(out), int(x.shape[0]), int(x.shape[1]),
                                        sm)
    _check(rc, "moe_decode_reduce_residual")


class MoEDecode:
    """One MoE block shape bound to the current CUDA device (owns a workspace).

    two_stream=False (default): router kernel, one expert kernel (shared
    and routed experts) and the combine on the main stream.  two_stream=True:
    MOE_FLAG_TWO_STREAM, the shared expert on the aux stream.  tcgen05=True:
    MOE_FLAG_TCGEN05, the expert kernel on tcgen05 with TMEM accumulators.
    fp8=True: MOE_FLAG_FP8_WEIGHTS (forward_fp8).  partial=True:
    MOE_FLAG_PARTIAL_SUM, `out` receives the fp32 expert sum without the
    residual (one tensor-parallel rank's share; see tp.py)."""

    def __init__(self, hidden: int, n_experts: int, top_k: int, inter: int, shared_inter: int = 0,
                 n_shared: int = 1, max_batch: int = 64, router_bias=None, two_stream: bool = False,
                 tcgen05: bool = False, extra_flags: int = 0, fp8: bool = False, partial: bool = False):
        self._lib = load_library()
        self._bias = router_bias  # keep the device tensor alive
        self.two_stream = bool(two_stream)
        self.tcgen05 = bool(tcgen05)
        flags = (MOE_FLAG_TWO_STREAM if two_stream else 0) | (MOE_FLAG_TCGEN05 if tcgen05 else 0) | int(extra_flags)
        flags |= MOE_FLAG_FP8_WEIGHTS if fp8 else 0
        flags |= MOE_FLAG_PARTIAL_SUM if partial else 0
        self.shapes = Shapes(hidden, n_experts, top_k, inter, shared_inter if n_shared else 0, n_shared,
                             max_batch, _ptr(router_bias), flags)
        h = ctypes.c_void_p()
        _check(self._lib.moe_decode_init(ctypes.byref(self.shapes), ctypes.byref(h)), "moe_decode_init")
        self._h = h
        self._aux = None
        self._tables = {}

    # -- pointer tables -------------------------------------------------------
    def _table(self, w: Union[Sequence, "object"]):
        """Host array of n_experts device pointers from a [E, ...] tensor or a list."""
        E = self.shapes.n_experts
        if hasattr(w, "data_ptr") and getattr(w, "dim", lambda: 0)() >= 3:
            key = ("t", w.data_ptr(), tuple(w.shape), tuple(w.stride()))
            arr = self._tables.get(key)
            if arr is None:
                if w.shape[0] != E:
                    raise ValueError(f"expected {E} experts, got {w.shape[0]}")
                base, step = w.data_ptr(), w.stride(0) * w.element_size()
                arr = (ctypes.c_void_p * E)(*[base + e * step for e in range(E)])
                if len(self._tables) > 8:
                    self._tables.clear()
                self._tables[key] = arr
            return arr
        ptrs = [_ptr(t) for t in w]
        if len(ptrs) != E:
            raise ValueError(f"expected {E} expert pointers, got {len(ptrs)}")
        return (ctypes.c_void_p * E)(*ptrs)

    def aux_stream(self):
        import torch
        if self._aux is None:
            self._aux = torch.cuda.Stream()
        return self._aux

    # -- entry points ---------------------------------------------------------
    def forward(self, x, router_w, w13, w2, shared_w13, shared_w2, out, topk_ids, topk_w,
                batch: Optional[int] = None, stream_main=None, stream_aux=None):
        """Enqueue one forward (device tensors).  Streams default to the current
        torch stream (main) and this object's side stream (aux)."""
        import torch
        if batch is None:
            batch = x.shape[0]
        sm = _stream_handle(stream_main if stream_main is not None else torch.cuda.current_stream())
        sa = _stream_handle(stream_aux if stream_aux is not None else self.aux_stream())
        rc = self._lib.moe_decode_forward(self._h, _ptr(x), _ptr(router_w), self._table(w13), self._table(w2),
                                          _ptr(shared_w13), _ptr(shared_w2), _ptr(out), _ptr(topk_ids),
                                          _ptr(topk_w), int(batch), sm, sa)
        _check(rc, "moe_decode_forward")

    def forward_fp8(self, x, router_w, w13q, w13s, w2q, w2s, shared_w13q, shared_w13s, shared_w2q, shared_w2s,
                    out, topk_ids, topk_w, batch: Optional[int] = None, stream_main=None, stream_aux=None):
        """Enqueue one forward with e4m3 expert weights (handle made with
        fp8=True): w13q/w2q [E, out, in] uint8 codes (or lists), w13s/w2s
        their float32 block scales [E, ceil(in/128), padded ceil(out/128)]."""
        import torch
        if batch is None:
            batch = x.shape[0]
        sm = _stream_handle(stream_main if stream_main is not None else torch.cuda.current_stream())
        sa = _stream_handle(stream_aux if stream_aux is not None else self.aux_stream())
        rc = self._lib.moe_decode_forward_fp8(self._h, _ptr(x), _ptr(router_w), self._table(w13q), self._table(w13s),
                                              self._table(w2q), self._table(w2s), _ptr(shared_w13q),
                                              _ptr(shared_w13s), _ptr(shared_w2q), _ptr(shared_w2s), _ptr(out),
                                              _ptr(topk_ids), _ptr(topk_w), int(batch), sm, sa)
        _check(rc, "moe_decode_forward_fp8")

    def forward_host(self, x_host, router_w, w13, w2, shared_w13, shared_w2, out_host, ids_host, w_host,
                     batch: Optional[int] = None, stream_main=None, stream_aux=None):
        """Host-buffer variant, synchronising stream_main: x is copied in; out/ids/w
        are stored by the kernels directly when all three are pinned (mapped)
        host tensors, else staged on the device and copied back."""
        import torch
        if batch is None:
            batch = x_host.shape[0]
        sm = _stream_handle(stream_main if stream_main is not None else torch.cuda.current_stream())
        sa = _stream_handle(stream_aux if stream_aux is not None else self.aux_stream())
        rc = self._lib.moe_decode_forward_host(self._h, _ptr(x_host), _ptr(router_w), self._table(w13),
                                               self._table(w2), _ptr(shared_w13), _ptr(shared_w2),
                                               _ptr(out_host), _ptr(ids_host), _ptr(w_host), int(batch), sm, sa)
        _check(rc, "moe_decode_forward_host")

    def set_timing_events(self, events):
        """Record per-kernel CUDA events in every forward (list of 6
        torch.cuda.Event(enable_timing=True)), or stop with None."""
        if events is None:
            _check(self._lib.moe_decode_set_timing_events(self._h, None, 0), "moe_decode_set_timing_events")
            self._events = None
            return
        if len(events) != MOE_TIMING_EVENTS:
            raise ValueError(f"need {MOE_TIMING_EVENTS} events")
        for ev in events:
            ev.record()  # materialise the underlying cudaEvent_t
        arr = (ctypes.c_void_p * MOE_TIMING_EVENTS)(*[ev.cuda_event for ev in events])
        self._events = events
        _check(self._lib.moe_decode_set_timing_events(self._h, arr, MOE_TIMING_EVENTS),
               "moe_decode_set_timing_events")

    def status(self) -> int:
        """Wait for the handle's work and return the device status (MOE_OK or an
        MOE_ERR_* code)."""
        return self._lib.moe_decode_get_status(self._h)

    def set_wait_limit(self, probes: int = 0):
        """Bound of the kernels' device-side waits in probes (0: the default)."""
        _check(self._lib.moe_decode_set_wait_limit(self._h, int(probes)), "moe_decode_set_wait_limit")

    def stats(self) -> dict:
        s = Stats()
        _check(self._lib.moe_decode_get_stats(self._h, ctypes.byref(s)), "moe_decode_get_stats")
        return {"forwards": s.forwards, "kernels_launched": s.kernels_launched, "last_kernels": s.last_kernels,
                "last_token_tiles": s.last_token_tiles, "stages_up": list(s.stages_up),
                "stages_down": list(s.stages_down)}

    def close(self):
        if getattr(self, "_h", None):
            self._lib.moe_decode_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
