"""fp64 CPU oracle of the MoE decode block -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never uses it and
shares no code with it.

Two independent implementations of the same definition:

* ``moe_oracle.c`` (plain C loops, fp64, OpenMP), loaded through ctypes here;
* ``moe_oracle_np.py`` (numpy fp64 restatement, small shapes).

All array arguments are numpy arrays of bf16 *bit patterns* (``uint16``),
row-major: x [B,H], router_w [H,E], w13[e] [H,2I], w2[e] [I,H],
sw13 [H,2Is], sw2 [Is,H]; the optional bias is float32 [E].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

from . import moe_oracle_np as np_oracle  # noqa: F401  (re-export)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_ERRORS = {-1: "bad argument", -2: "a selected expert has no weights", -3: "out of memory"}


def build_c_oracle(force: bool = False) -> str:
    """Compile moe_oracle.c into oracle/liboracle.so with gcc (-O2 -fopenmp)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build_c_oracle()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_router.argtypes = [P, P, P, I, I, I, I, P, P, P]
        lib.oracle_router.restype = I
        lib.oracle_block.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P]
        lib.oracle_block.restype = I
        lib.oracle_expert_outputs.argtypes = [P, I, I, P, P, I, I, P, P]
        lib.oracle_expert_outputs.restype = I
        lib.oracle_combine.argtypes = [P, P, P, P, I, I, I, P]
        lib.oracle_combine.restype = I
        lib.oracle_expert_outputs_fp8.argtypes = [P, I, I, P, P, P, P, I, I, P, P]
        lib.oracle_expert_outputs_fp8.restype = I
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bf16 bit patterns, got {a.dtype}")
    return a


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what}: oracle error {rc} ({_ERRORS.get(rc, 'unknown')})")


def router(x, router_w, k: int, bias=None):
    """Steps 1-4 (C oracle).  Returns (logits [B,E] f64, ids [B,k] i32, w [B,k] f64)."""
    lib = _load()
    x = _u16(x)
    router_w = _u16(router_w)
    B, H = x.shape
    H2, E = router_w.shape
    assert H == H2
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    logits = np.zeros((B, E), np.float64)
    ids = np.zeros((B, k), np.int32)
    w = np.zeros((B, k), np.float64)
    _check(lib.oracle_router(_ptr(x), _ptr(router_w), _ptr(b), B, H, E, k,
                             _ptr(logits), _ptr(ids), _ptr(w)), "oracle_router")
    return logits, ids, w


def block(x, ids, w, w13: Sequence, w2: Sequence, sw13=None, sw2=None, n_experts=None):
    """Steps 5-7 (C oracle) for a given routing.  ``w13``/``w2`` are sequences of
    length E (entries for experts that are never selected may be None)."""
    lib = _load()
    x = _u16(x)
    B, H = x.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    k = ids.shape[1] if ids.ndim == 2 else 0
    E = len(w13) if n_experts is None else n_experts
    keep = []
    arr13 = (ctypes.c_void_p * E)()
    arr2 = (ctypes.c_void_p * E)()
    inter = None
    for e in range(E):
        if w13[e] is not None:
            a13 = _u16(w13[e]); a2 = _u16(w2[e])
            keep += [a13, a2]
            arr13[e] = a13.ctypes.data
            arr2[e] = a2.ctypes.data
            inter = a13.shape[1] // 2
    if inter is None:
        raise ValueError("no expert weights given")
    n_shared = 0 if sw13 is None else 1
    Is = 0
    if n_shared:
        sw13 = _u16(sw13); sw2 = _u16(sw2)
        Is = sw13.shape[1] // 2
    out = np.zeros((B, H), np.float64)
    _check(lib.oracle_block(_ptr(x), _ptr(ids), _ptr(w), arr13, arr2, _ptr(sw13), _ptr(sw2),
                            B, H, E, k, inter, Is, n_shared, _ptr(out)), "oracle_block")
    del keep
    return out


def expert_outputs(x, w13e, w2e, rows):
    """Step 5 for one expert (C oracle): y [len(rows), H] f64, row i the
    SwiGLU MLP of token rows[i] through that expert's w13e [H,2I], w2e [I,H]."""
    lib = _load()
    x = _u16(x)
    B, H = x.shape
    w13e = _u16(w13e)
    w2e = _u16(w2e)
    I = w13e.shape[1] // 2
    assert w13e.shape == (H, 2 * I) and w2e.shape == (I, H)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    y = np.zeros((len(rows), H), np.float64)
    _check(lib.oracle_expert_outputs(_ptr(x), B, H, _ptr(w13e), _ptr(w2e), I, len(rows), _ptr(rows), _ptr(y)),
           "oracle_expert_outputs")
    return y


def block_streamed(x, ids, w, fetch_expert, sw13=None, sw2=None):
    """Steps 5-7 like ``block``, holding one expert's weights at a time:
    ``fetch_expert(e)`` returns (w13[e], w2[e]) as bf16 bit arrays and is
    called once per distinct selected expert, in ascending id order.  Each
    expert's MLP is evaluated for the tokens that chose it, the per-assignment
    outputs are kept, and the sum of step 7 is taken in the same order as
    ``block`` (residual, then j = 0..k-1, then the shared expert), so the
    result is bitwise equal to ``block``'s."""
    lib = _load()
    x = _u16(x)
    B, H = x.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    k = ids.shape[1] if ids.ndim == 2 else 0
    y = np.zeros((B, k, H), np.float64)
    for e in sorted(set(ids.ravel().tolist())):
        bj = np.argwhere(ids == e)  # (token, slot) pairs that chose e
        a13, a2 = fetch_expert(e)
        y[bj[:, 0], bj[:, 1]] = expert_outputs(x, a13, a2, bj[:, 0])
        del a13, a2
    s = None
    if sw13 is not None:
        s = expert_outputs(x, sw13, sw2, np.arange(B))
    out = np.zeros((B, H), np.float64)
    _check(lib.oracle_combine(_ptr(x), _ptr(w), _ptr(y), _ptr(s), B, H, k, _ptr(out)), "oracle_combine")
    return out


def e4m3_value(code: int) -> float:
    """The fp64 value of an 8-bit e4m3 code (NaN for the NaN codes)."""
    return float(_load().oracle_e4m3_value(int(code) & 0xFF))


def expert_outputs_fp8(x, q13, s13, q2, s2, rows):
    """Step 5 for one expert with block-scaled e4m3 weights (C oracle):
    q13 uint8 [2I, H] with fp32 scales [ceil(2I/128), ceil(H/128)], q2 uint8
    [H, I] with scales [ceil(H/128), ceil(I/128)]; y [len(rows), H] f64."""
    lib = _load()
    x = _u16(x)
    B, H = x.shape
    q13 = np.ascontiguousarray(q13, dtype=np.uint8)
    q2 = np.ascontiguousarray(q2, dtype=np.uint8)
    s13 = np.ascontiguousarray(s13, dtype=np.float32)
    s2 = np.ascontiguousarray(s2, dtype=np.float32)
    I = q13.shape[0] // 2
    assert q13.shape == (2 * I, H) and q2.shape == (H, I)
    assert s13.shape == (-(-2 * I // 128), -(-H // 128)) and s2.shape == (-(-H // 128), -(-I // 128))
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    y = np.zeros((len(rows), H), np.float64)
    _check(lib.oracle_expert_outputs_fp8(_ptr(x), B, H, _ptr(q13), _ptr(s13), _ptr(q2), _ptr(s2), I, len(rows),
                                         _ptr(rows), _ptr(y)), "oracle_expert_outputs_fp8")
    return y


def block_streamed_fp8(x, ids, w, fetch_expert, shared=None):
    """Steps 5-7 with block-scaled e4m3 expert weights, one expert at a time:
    ``fetch_expert(e)`` returns (q13, s13, q2, s2); ``shared`` is the shared
    expert's (q13, s13, q2, s2) or None.  The sum of step 7 is taken in the
    same order as ``block``."""
    lib = _load()
    x = _u16(x)
    B, H = x.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    k = ids.shape[1] if ids.ndim == 2 else 0
    y = np.zeros((B, k, H), np.float64)
    for e in sorted(set(ids.ravel().tolist())):
        bj = np.argwhere(ids == e)
        y[bj[:, 0], bj[:, 1]] = expert_outputs_fp8(x, *fetch_expert(e), bj[:, 0])
    s = None if shared is None else expert_outputs_fp8(x, *shared, np.arange(B))
    out = np.zeros((B, H), np.float64)
    _check(lib.oracle_combine(_ptr(x), _ptr(w), _ptr(y), _ptr(s), B, H, k, _ptr(out)), "oracle_combine")
    return out


def moe_forward(x, router_w, w13, w2, sw13, sw2, k: int, bias=None):
    """Steps 1-7 (C oracle).  Returns (out [B,H] f64, ids, w, logits)."""
    logits, ids, w = router(x, router_w, k, bias)
    out = block(x, ids, w, w13, w2, sw13, sw2)
    return out, ids, w, logits


def topk_margin(logits: np.ndarray, k: int) -> np.ndarray:
    """Smallest gap between consecutive sorted logits among each row's top k+1
    (used by tests to reject inputs whose top-k order is not well separated)."""
    s = -np.sort(-logits, axis=1)[:, : k + 1]
    return np.min(s[:, :-1] - s[:, 1:], axis=1)
