"""fp64 CPU oracle of one MoE decode-layer step (ctypes wrapper of moe_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are its only callers. The product path (the
CUDA library and its binding) never imports this package, and this package
never imports the product. The only code the two sides share is the seeded
input generator package ``synth``.

Parity status of each function is recorded in the test suite
(``tests/test_oracle_pins.py``): every stage is pinned by closed forms,
library special cases, invariants or brute force on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "libmoe_oracle.so")
# the same source compiled with its planted mistakes (the pins' own test only)
MUTANT_LIB = os.path.join(_HERE, "libmoe_oracle_mutants.so")

OK, EINVAL, EMISSING, ENONFINITE = 0, -1, -2, -3


def build(verbose: bool = False) -> None:
    src = os.path.join(_HERE, "moe_oracle.c")
    for out, extra in ((LIB, []), (MUTANT_LIB, ["-DORACLE_MUTANTS"])):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", *extra, "-o", out, src, "-lm"]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True, cwd=_HERE)


class _Dims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
                ("I", ctypes.c_int), ("Is", ctypes.c_int), ("eps", ctypes.c_double)]


class _Weights(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("w_gate", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("ws_gate", ctypes.c_void_p), ("ws_up", ctypes.c_void_p),
                ("ws_down", ctypes.c_void_p)]


_libs = {}
_active = LIB


def _load(path):
    if path not in _libs:
        if not os.path.exists(path):
            build()
        lib = ctypes.CDLL(path)
        vp, i, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        if path == MUTANT_LIB:
            lib.oracle_set_mutant.argtypes = [i]
            lib.oracle_set_mutant.restype = None
        lib.oracle_bf16_round.argtypes = [d]
        lib.oracle_bf16_round.restype = d
        lib.oracle_double_to_bf16_bits.argtypes = [d]
        lib.oracle_double_to_bf16_bits.restype = ctypes.c_uint16
        lib.oracle_rmsnorm.argtypes = [i, d, vp, vp, vp]
        lib.oracle_rmsnorm.restype = None
        lib.oracle_router.argtypes = [i, i, vp, vp, vp, vp]
        lib.oracle_router.restype = None
        lib.oracle_topk.argtypes = [i, i, vp, vp]
        lib.oracle_topk.restype = i
        lib.oracle_softmax_selected.argtypes = [i, vp, vp, vp]
        lib.oracle_softmax_selected.restype = None
        lib.oracle_swiglu.argtypes = [i, i, vp, vp, vp, vp, vp]
        lib.oracle_swiglu.restype = None
        lib.oracle_layer.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), i, vp,
                                     vp, vp, vp, vp, vp]
        lib.oracle_layer.restype = i
        lib.oracle_layer_selected.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), i, vp,
                                              vp, vp, vp, vp, vp, vp]
        lib.oracle_layer_selected.restype = i
        lib.oracle_layer_partial.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Weights), i, vp, vp, i, i, i,
                                             vp]
        lib.oracle_layer_partial.restype = i
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = d
        lib.oracle_dequant_e4m3.argtypes = [i, i, vp, vp, vp]
        lib.oracle_dequant_e4m3.restype = i
        _libs[path] = lib
    return _libs[path]


def _L():
    return _load(_active)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data


MUTANTS = {
    1: "no_n_round", 2: "no_h_round", 3: "residual_n", 4: "ties_high", 5: "equal_weights",
    6: "no_shared", 7: "silu_on_up", 8: "no_gamma", 9: "down_transposed", 10: "no_bias",
    11: "eps_outside", 12: "e4m3_bias", 13: "block_transposed",
}


def set_mutant(m: int) -> None:
    """Swap in one planted mistake (tests of the pins only): every later call runs the
    separately compiled mutant build with mistake m. 0 restores the oracle itself."""
    global _active
    if int(m) == 0:
        if MUTANT_LIB in _libs:
            _libs[MUTANT_LIB].oracle_set_mutant(0)
        _active = LIB
    else:
        _load(MUTANT_LIB).oracle_set_mutant(int(m))
        _active = MUTANT_LIB


# ---- single stages ---------------------------------------------------------------

def bf16_round(v: float) -> float:
    return _L().oracle_bf16_round(float(v))


def bf16_bits(v: float) -> int:
    return int(_L().oracle_double_to_bf16_bits(float(v)))


def rmsnorm(x_bits: np.ndarray, gamma_bits: np.ndarray, eps: float) -> np.ndarray:
    x, g = _c(x_bits, np.uint16), _c(gamma_bits, np.uint16)
    out = np.empty(x.shape[0], dtype=np.float64)
    _L().oracle_rmsnorm(x.shape[0], eps, _p(x), _p(g), _p(out))
    return out


def router(n: np.ndarray, w_router_bits: np.ndarray, bias=None) -> np.ndarray:
    n, w = _c(n, np.float64), _c(w_router_bits, np.uint16)
    b = None if bias is None else _c(bias, np.float32)
    E, H = w.shape
    out = np.empty(E, dtype=np.float64)
    _L().oracle_router(H, E, _p(n), _p(w), _p(b), _p(out))
    return out


def topk(values: np.ndarray, k: int) -> np.ndarray:
    """k largest values, ties to the lower index, in descending order. fp32 inputs
    (e.g. GPU logits) are widened exactly, so comparisons are the fp32 ones."""
    v = _c(values, np.float64)
    idx = np.empty(k, dtype=np.int32)
    rc = _L().oracle_topk(v.shape[0], k, _p(v), _p(idx))
    if rc != 0:
        raise ValueError("oracle_topk: non-finite value or bad k")
    return idx


def softmax_selected(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    lg, ix = _c(logits, np.float64), _c(idx, np.int32)
    out = np.empty(ix.shape[0], dtype=np.float64)
    _L().oracle_softmax_selected(ix.shape[0], _p(lg), _p(ix), _p(out))
    return out


def swiglu(n: np.ndarray, wg_bits, wu_bits, wd_bits) -> np.ndarray:
    n = _c(n, np.float64)
    wg, wu, wd = _c(wg_bits, np.uint16), _c(wu_bits, np.uint16), _c(wd_bits, np.uint16)
    F, H = wg.shape
    out = np.empty(H, dtype=np.float64)
    _L().oracle_swiglu(H, F, _p(n), _p(wg), _p(wu), _p(wd), _p(out))
    return out


# ---- FP8 expert weights ----------------------------------------------------------------

def e4m3_value(code: int) -> float:
    return _L().oracle_e4m3_to_double(int(code))


def dequant_e4m3(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """bf16 bits of value(code) * scale of its 128 x 128 block ([rows, cols] codes,
    [ceil(rows/128), ceil(cols/128)] scales); raises if a product is not a bf16 value."""
    q = _c(codes, np.uint8)
    rows, cols = q.shape
    sc = _c(scales, np.float32)
    out = np.empty((rows, cols), dtype=np.uint16)
    if _L().oracle_dequant_e4m3(rows, cols, _p(q), _p(sc), _p(out)) != OK:
        raise ValueError("oracle_dequant_e4m3: a dequantised weight is not a bf16 value")
    return out


def fp8_expert(fp8: dict):
    """(W_g, W_u, W_d) bf16 bits of an expert given as {gate, up, down: (codes, scales)}."""
    return tuple(dequant_e4m3(*fp8[m]) for m in ("gate", "up", "down"))


# ---- whole layer -------------------------------------------------------------------

def layer(dims: dict, weights: dict, x_bits: np.ndarray, selection=None) -> dict:
    """Run the oracle on rows x_bits [B, H].

    dims: H, E, k, I, Is, eps.  weights: gamma [H], w_router [E,H], router_bias
    [E] or None, experts {e: (W_g [I,H], W_u [I,H], W_d [H,I])} (only the
    experts the rows select need be present), ws_gate [Is,H], ws_up [Is,H],
    ws_down [H,Is]; all bf16 bit arrays. Returns logits, idx, w, y_pre, y.

    selection: None (each row takes the top-k of its logits), or int [B, k] -- each
    row's k distinct experts given (oracle_layer_selected: the weights are the
    softmax of the row's own logits over the given set).
    """
    H, E, k = dims["H"], dims["E"], dims["k"]
    x = _c(x_bits, np.uint16).reshape(-1, H)
    B = x.shape[0]
    sel = None
    if selection is not None:
        sel = _c(selection, np.int32).reshape(B, k)
    keep = []  # keep arrays alive across the call
    d, w = _structs(dims, weights, keep)
    logits = np.empty((B, E), dtype=np.float64)
    idx = np.empty((B, k), dtype=np.int32)
    wts = np.empty((B, k), dtype=np.float64)
    y_pre = np.empty((B, H), dtype=np.float64)
    y = np.empty((B, H), dtype=np.uint16)
    if sel is None:
        rc = _L().oracle_layer(ctypes.byref(d), ctypes.byref(w), B, _p(x), _p(logits), _p(idx),
                               _p(wts), _p(y_pre), _p(y))
    else:
        rc = _L().oracle_layer_selected(ctypes.byref(d), ctypes.byref(w), B, _p(x), _p(sel), _p(logits),
                                        _p(idx), _p(wts), _p(y_pre), _p(y))
    if rc != OK:
        raise RuntimeError(f"oracle_layer failed: {rc}")
    return {"logits": logits, "idx": idx, "w": wts, "y_pre": y_pre, "y": y}


def layer_partial(dims: dict, weights: dict, x_bits: np.ndarray, e0: int, e1: int, with_rs: bool,
                  selection=None) -> np.ndarray:
    """The part of the layer's output (fp64 [B, H], unrounded) that experts e0 <= e < e1
    contribute, plus x + s when with_rs (oracle_layer_partial). Summed over a partition
    of the experts with with_rs set for one part, it is layer(...)["y_pre"]. weights as
    for layer; only the experts in the range need be present. selection: as for layer."""
    H, k = dims["H"], dims["k"]
    x = _c(x_bits, np.uint16).reshape(-1, H)
    B = x.shape[0]
    sel = None if selection is None else _c(selection, np.int32).reshape(B, k)
    keep = []
    d, w = _structs(dims, weights, keep)
    out = np.empty((B, H), dtype=np.float64)
    rc = _L().oracle_layer_partial(ctypes.byref(d), ctypes.byref(w), B, _p(x), None if sel is None else _p(sel),
                                   int(e0), int(e1), 1 if with_rs else 0, _p(out))
    if rc != OK:
        raise RuntimeError(f"oracle_layer_partial failed: {rc}")
    return out


def _structs(dims: dict, weights: dict, keep: list):
    """The C structs of dims and weights (arrays kept alive in keep)."""
    E = dims["E"]

    def arr(a, dt):
        a2 = _c(a, dt)
        keep.append(a2)
        return a2

    gp = (ctypes.c_void_p * E)()
    up = (ctypes.c_void_p * E)()
    dp = (ctypes.c_void_p * E)()
    for e, (g, u, d) in weights["experts"].items():
        gp[e] = arr(g, np.uint16).ctypes.data
        up[e] = arr(u, np.uint16).ctypes.data
        dp[e] = arr(d, np.uint16).ctypes.data
    bias = weights.get("router_bias")
    w = _Weights(
        gamma=arr(weights["gamma"], np.uint16).ctypes.data,
        w_router=arr(weights["w_router"], np.uint16).ctypes.data,
        router_bias=None if bias is None else arr(bias, np.float32).ctypes.data,
        w_gate=ctypes.cast(gp, ctypes.c_void_p), w_up=ctypes.cast(up, ctypes.c_void_p),
        w_down=ctypes.cast(dp, ctypes.c_void_p),
        ws_gate=arr(weights["ws_gate"], np.uint16).ctypes.data,
        ws_up=arr(weights["ws_up"], np.uint16).ctypes.data,
        ws_down=arr(weights["ws_down"], np.uint16).ctypes.data)
    keep.append((gp, up, dp))
    d = _Dims(H=dims["H"], E=E, k=dims["k"], I=dims["I"], Is=dims["Is"], eps=float(dims["eps"]))
    return d, w


def workload_layer(wl, layer_index: int, x_bits: np.ndarray, shared=None, w_router=None,
                   selection=None, fp8: bool = False) -> dict:
    """Oracle of one layer of a ``synth.Workload`` on rows x_bits [B, H].

    Only the experts that the rows select are regenerated on the host (one row
    at a time, so host memory stays at 16 experts). ``shared`` and ``w_router``
    may be passed in to avoid regenerating them for every call. ``selection``
    (int [B, k], optional) gives each row's experts instead of its top-k. ``fp8``: the
    experts are the workload's FP8 ones (E4M3 codes and block scales, dequantised).
    """
    dims = dict(H=wl.H, E=wl.E, k=wl.k, I=wl.I, Is=wl.Is, eps=wl.eps)
    gamma = wl.gamma_host(layer_index)
    wr = wl.w_router_host(layer_index) if w_router is None else w_router
    bias = wl.bias_host(layer_index)
    sg, su, sd = wl.shared_host(layer_index) if shared is None else shared
    x = _c(x_bits, np.uint16).reshape(-1, wl.H)
    outs = []
    for b in range(x.shape[0]):
        if selection is None:
            n = rmsnorm(x[b], gamma, wl.eps)
            sel = topk(router(n, wr, bias), wl.k)
            given = None
        else:
            sel = given = np.asarray(selection[b], dtype=np.int32).reshape(1, wl.k)
        experts = {int(e): (fp8_expert(wl.expert_fp8_host(layer_index, int(e))) if fp8
                            else wl.expert_host(layer_index, int(e))) for e in np.ravel(sel)}
        outs.append(layer(dims, dict(gamma=gamma, w_router=wr, router_bias=bias, experts=experts,
                                     ws_gate=sg, ws_up=su, ws_down=sd), x[b:b + 1], selection=given))
        del experts
    return {key: np.concatenate([o[key] for o in outs], axis=0) for key in outs[0]}
