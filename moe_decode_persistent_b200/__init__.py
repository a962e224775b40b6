"""Python binding of the B200 persistent MoE decode-layer step (include/moe_decode.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libmoe_decode.so``. There is no CPU or PyTorch fallback; constructing a
``MoeDecode`` without the built library or without a B200 raises.

PyTorch is used by callers for device memory and streams; this module accepts
either torch tensors or raw device pointers (ints).
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(_HERE)
LIB = os.path.join(_HERE, "libmoe_decode.so")
# the same sources built with every schedule-derived index range-checked (MOE_BOUNDS_CHECK):
# a test build, standing in for a memory checker
CHECKED_LIB = os.path.join(_HERE, "libmoe_decode_checked.so")
HEADER = os.path.join(ROOT, "include", "moe_decode.h")
SOURCES = [os.path.join(_HERE, "csrc", f)
           for f in ("moe_decode_kernel.cu", "moe_decode_api.cu", "moe_decode_noalloc.cu")]

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_ARCH = -2
MOE_ERR_UNSUPPORTED_SHAPE = -3
MOE_ERR_COOPERATIVE = -4
MOE_ERR_CUDA = -5
MOE_ERR_TIMEOUT = -6
MOE_ERR_NONFINITE = -7
MOE_ERR_NO_MEMORY = -8
MOE_ERR_BOUNDS = -9

DEBUG_JITTER = 1
DEBUG_WITHHOLD_NREADY = 2
DEBUG_BAD_SLOT = 4  # bounds-checked build only

PATH_CUDA_CORE = 0
PATH_TENSOR_CORE = 1


def nvcc_command(out: str = LIB, checked: bool = False) -> list[str]:
    return ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
            "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            *(["-DMOE_BOUNDS_CHECK"] if checked else []),
            "-I" + os.path.join(ROOT, "include"), "-o", out, *SOURCES]


def build(verbose: bool = False) -> None:
    """Compile libmoe_decode.so and the bounds-checked libmoe_decode_checked.so in-tree
    for sm_100a (the two nvcc runs in parallel)."""
    cmds = [nvcc_command(), nvcc_command(CHECKED_LIB, checked=True)]
    procs = []
    for cmd in cmds:
        if verbose:
            print(" ".join(cmd))
        procs.append(subprocess.Popen(cmd, cwd=_HERE))
    for cmd, pr in zip(cmds, procs):
        if pr.wait() != 0:
            raise subprocess.CalledProcessError(pr.returncode, cmd)


def declared_symbols() -> list[str]:
    """Function names declared by include/moe_decode.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(moe_decode_[a-z0-9_]+)\s*\(", text)))


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k_max", ctypes.c_int),
                ("inter", ctypes.c_int), ("shared_inter", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("n_layers", ctypes.c_int), ("eps", ctypes.c_float)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("w_gate", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("ws_gate", ctypes.c_void_p), ("ws_up", ctypes.c_void_p),
                ("ws_down", ctypes.c_void_p)]


class LayerWeightsFp8(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("w_gate", ctypes.c_void_p),
                ("w_gate_scale", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_up_scale", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("w_down_scale", ctypes.c_void_p), ("ws_gate", ctypes.c_void_p),
                ("ws_up", ctypes.c_void_p), ("ws_down", ctypes.c_void_p)]


# keys of a layer mapping with FP8 experts (synth.Workload.device_layer_fp8) per field
_FP8_KEYS = {"w_gate": "w_gate_q", "w_up": "w_up_q", "w_down": "w_down_q"}


class Debug(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p),
                ("topk_w", ctypes.c_void_p), ("n_unique", ctypes.c_void_p)]


_lib = None
_checked_lib = None


def lib(checked: bool = False):
    """The loaded C-ABI library (raises if it has not been built); checked: the
    bounds-checked build."""
    global _lib, _checked_lib
    if checked:
        if _checked_lib is None:
            _checked_lib = _load(CHECKED_LIB)
        return _checked_lib
    if _lib is None:
        _lib = _load(LIB)
    return _lib


def _load(path):
    if True:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with moe_decode_persistent_b200.build()")
        L = ctypes.CDLL(path)
        vp, i, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
        L.moe_decode_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LayerWeights), i,
                                        ctypes.POINTER(vp)]
        L.moe_decode_create.restype = i
        L.moe_decode_create_fp8.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LayerWeightsFp8), i,
                                            ctypes.POINTER(vp)]
        L.moe_decode_create_fp8.restype = i
        L.moe_decode_step.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.moe_decode_step.restype = i
        L.moe_decode_step_host.argtypes = [vp, vp, vp, i, i, vp, vp]
        L.moe_decode_step_host.restype = i
        L.moe_decode_get_status.argtypes = [vp, ctypes.POINTER(i)]
        L.moe_decode_get_status.restype = i
        L.moe_decode_launches_per_step.argtypes = [vp]
        L.moe_decode_launches_per_step.restype = i
        L.moe_decode_set_trace.argtypes = [vp, vp]
        L.moe_decode_set_trace.restype = i
        L.moe_decode_trace_slots.argtypes = [vp]
        L.moe_decode_trace_slots.restype = i
        L.moe_decode_set_debug.argtypes = [vp, u, u]
        L.moe_decode_set_debug.restype = i
        L.moe_decode_set_tc_min_batch.argtypes = [vp, i]
        L.moe_decode_set_tc_min_batch.restype = i
        L.moe_decode_step_path.argtypes = [vp, i]
        L.moe_decode_step_path.restype = i
        L.moe_decode_destroy.argtypes = [vp]
        L.moe_decode_destroy.restype = None
        L.moe_decode_step_noalloc.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LayerWeights),
                                              vp, vp, i, i, vp, vp]
        L.moe_decode_step_noalloc.restype = i
        L.moe_decode_create_ep.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LayerWeights), i, i, i,
                                           ctypes.POINTER(vp)]
        L.moe_decode_create_ep.restype = i
        L.moe_decode_step_partial.argtypes = [vp, vp, vp, i, i, i, vp, vp]
        L.moe_decode_step_partial.restype = i
        L.moe_decode_partial_to_bf16.argtypes = [vp, vp, ctypes.c_longlong, i, vp]
        L.moe_decode_partial_to_bf16.restype = i
        L.moe_decode_strerror.argtypes = [i]
        L.moe_decode_strerror.restype = ctypes.c_char_p
    return L


def strerror(code: int) -> str:
    return lib().moe_decode_strerror(int(code)).decode()


def partial_to_bf16(part, out, device: int = 0, stream=None) -> None:
    """out <- bf16(part) elementwise (device fp32 -> device bf16, same element count),
    asynchronous on `stream`: the output of an expert-parallel step once the ranks'
    partials are summed."""
    n = int(part.numel())
    if int(out.numel()) != n or str(part.dtype) != "torch.float32":
        raise ValueError("partial_to_bf16: fp32 input and an output of the same element count")
    _check(lib().moe_decode_partial_to_bf16(_ptr(part), _ptr(out), n, int(device), _stream_handle(stream)),
           "moe_decode_partial_to_bf16")


class MoeDecodeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} ({code})")
        self.code = code


def _check(code: int, what: str) -> None:
    if code != MOE_OK:
        raise MoeDecodeError(code, what)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


_ROW_DTYPES = ("torch.bfloat16", "torch.int16", "torch.uint16")  # bf16 values or their bit patterns


def _check_rows(t, name: str, batch: int, hidden: int, device_type: str, what: str) -> None:
    """A torch tensor given as a row buffer must hold bf16 values (or their bit patterns
    as int16/uint16), be contiguous, live on `device_type` ("cuda" or "cpu") and hold at
    least batch x hidden elements; otherwise the call fails with MOE_ERR_INVALID_ARG
    before reaching the library. Raw pointers (ints) are not inspected."""
    if t is None or isinstance(t, int):
        return
    problem = None
    if str(t.dtype) not in _ROW_DTYPES:
        problem = f"dtype {t.dtype}, not bfloat16 (or its bits as int16/uint16)"
    elif t.device.type != device_type:
        problem = f"on {t.device.type}, not {device_type}"
    elif not t.is_contiguous():
        problem = "not contiguous"
    elif t.numel() < max(0, batch) * hidden:
        problem = f"{t.numel()} values for {batch} rows of {hidden}"
    if problem:
        raise MoeDecodeError(MOE_ERR_INVALID_ARG, f"{what}: {name} is {problem}")


def _stream_handle(stream) -> int | None:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def step_noalloc(hidden, n_experts, inter, shared_inter, layers, x, y, batch, top_k, eps=1e-6,
                 stream=None, device_status=None) -> None:
    """The decode step without a handle and without any device allocation (the
    library's built-in scratch; see moe_decode_step_noalloc in the header).

    For callers that cannot allocate device memory. Limits: batch <= 4, top_k <=
    16, hidden <= 7168, n_experts <= 1024, inter <= 1024, shared_inter <= 2048,
    at most 2 layers. Calls that overlap on the GPU race on the shared scratch.
    device_status (required): a zeroed device int32 that receives the first
    device-side MOE_ERR_* of the step.
    """
    for name, t in (("x", x), ("y", y)):
        _check_rows(t, name, batch, hidden, "cuda", "moe_decode_step_noalloc")
    cfg = Config(hidden, n_experts, top_k, inter, shared_inter, batch, len(layers), eps)
    arr = (LayerWeights * len(layers))()
    for i, w in enumerate(layers):
        arr[i] = LayerWeights(*(_ptr(w.get(name)) for name, _ in LayerWeights._fields_))
    _check(lib().moe_decode_step_noalloc(ctypes.byref(cfg), arr, _ptr(x), _ptr(y), int(batch), int(top_k),
                                         _stream_handle(stream), _ptr(device_status)),
           "moe_decode_step_noalloc")


class MoeDecode:
    """Handle of one configured decode layer stack on one device.

    layers: sequence of mappings with keys gamma, w_router, router_bias (or None),
    w_gate, w_up, w_down, ws_gate, ws_up, ws_down (torch tensors or device pointers).
    The caller keeps those tensors alive for the handle's lifetime. checked: run the
    bounds-checked build (libmoe_decode_checked.so), which reports a schedule-derived
    index outside its buffer as MOE_ERR_BOUNDS instead of accessing it.
    expert_range: (e0, e1) for one rank of an expert-parallel layer
    (moe_decode_create_ep): one layer whose w_gate / w_up / w_down hold only experts
    e0 .. e1 - 1; its steps go through step_partial.
    """

    def __init__(self, hidden, n_experts, top_k_max, inter, shared_inter, max_batch, layers,
                 eps=1e-6, device=0, checked=False, fp8=False, expert_range=None):
        self._lib = lib(checked)  # checked: the bounds-checked test build of the library
        self.cfg = Config(hidden, n_experts, top_k_max, inter, shared_inter, max_batch,
                          len(layers), eps)
        self._weights_keepalive = layers
        h = ctypes.c_void_p()
        if fp8:  # layers with FP8 experts: w_gate_q / w_gate_scale ... (moe_decode_create_fp8)
            arr = (LayerWeightsFp8 * len(layers))()
            for i, w in enumerate(layers):
                arr[i] = LayerWeightsFp8(*(_ptr(w.get(_FP8_KEYS.get(name, name))) for name, _ in LayerWeightsFp8._fields_))
            _check(self._lib.moe_decode_create_fp8(ctypes.byref(self.cfg), arr, int(device), ctypes.byref(h)),
                   "moe_decode_create_fp8")
        else:
            arr = (LayerWeights * len(layers))()
            for i, w in enumerate(layers):
                arr[i] = LayerWeights(*(_ptr(w.get(name)) for name, _ in LayerWeights._fields_))
            if expert_range is not None:
                e0, e1 = (int(v) for v in expert_range)
                _check(self._lib.moe_decode_create_ep(ctypes.byref(self.cfg), arr, int(device), e0, e1,
                                                      ctypes.byref(h)), "moe_decode_create_ep")
            else:
                _check(self._lib.moe_decode_create(ctypes.byref(self.cfg), arr, int(device), ctypes.byref(h)),
                       "moe_decode_create")
        self.handle = h
        self.n_layers = len(layers)

    def step(self, x, y, batch, top_k, stream=None, debug=None) -> None:
        """y <- layer stack(x); x, y device bf16 [batch, hidden]; asynchronous on `stream`."""
        for name, t in (("x", x), ("y", y)):
            _check_rows(t, name, batch, self.cfg.hidden, "cuda", "moe_decode_step")
        dbg = self._debug(debug)
        _check(self._lib.moe_decode_step(self.handle, _ptr(x), _ptr(y), int(batch), int(top_k),
                                     _stream_handle(stream), dbg), "moe_decode_step")

    def step_partial(self, x, y_part, batch, top_k, residual_shared=True, stream=None, debug=None) -> None:
        """y_part <- the fp32 partial output of a one-layer step over the handle's experts
        (x + shared expert included when residual_shared); x device bf16 and y_part device
        fp32, both [batch, hidden]."""
        _check_rows(x, "x", batch, self.cfg.hidden, "cuda", "moe_decode_step_partial")
        if str(y_part.dtype) != "torch.float32" or tuple(y_part.shape) != (batch, self.cfg.hidden) or \
                not y_part.is_contiguous() or y_part.device.type != "cuda":
            raise ValueError("moe_decode_step_partial: y_part must be a contiguous CUDA fp32 [batch, hidden] tensor")
        dbg = self._debug(debug)
        _check(self._lib.moe_decode_step_partial(self.handle, _ptr(x), _ptr(y_part), int(batch), int(top_k),
                                                 1 if residual_shared else 0, _stream_handle(stream), dbg),
               "moe_decode_step_partial")

    def step_host(self, x_host, y_host, batch, top_k, stream=None, debug=None) -> None:
        """Same step on host buffers (pinned torch CPU tensors or host pointers)."""
        for name, t in (("x_host", x_host), ("y_host", y_host)):
            _check_rows(t, name, batch, self.cfg.hidden, "cpu", "moe_decode_step_host")
        dbg = self._debug(debug)
        _check(self._lib.moe_decode_step_host(self.handle, _ptr(x_host), _ptr(y_host), int(batch),
                                          int(top_k), _stream_handle(stream), dbg),
               "moe_decode_step_host")

    def _debug(self, debug):
        if debug is None:
            return None
        arr = (Debug * self.n_layers)()
        for i, d in enumerate(debug):
            if d is not None:
                arr[i] = Debug(_ptr(d.get("logits")), _ptr(d.get("topk_idx")),
                               _ptr(d.get("topk_w")), _ptr(d.get("n_unique")))
        self._dbg_keepalive = (arr, debug)
        return ctypes.cast(arr, ctypes.c_void_p)

    def status(self) -> int:
        """Device status of the completed steps (MOE_OK or a MOE_ERR_* code); clears it."""
        v = ctypes.c_int(0)
        _check(self._lib.moe_decode_get_status(self.handle, ctypes.byref(v)), "moe_decode_get_status")
        return v.value

    def launches_per_step(self) -> int:
        return self._lib.moe_decode_launches_per_step(self.handle)

    def set_debug(self, flags: int, wait_ms: int = 2000) -> None:
        _check(self._lib.moe_decode_set_debug(self.handle, int(flags), int(wait_ms)), "moe_decode_set_debug")

    def set_tc_min_batch(self, min_batch: int) -> None:
        """Steps of at least min_batch rows take the tensor-core kernel (0: never)."""
        _check(self._lib.moe_decode_set_tc_min_batch(self.handle, int(min_batch)), "moe_decode_set_tc_min_batch")

    def step_path(self, batch: int) -> int:
        """PATH_CUDA_CORE or PATH_TENSOR_CORE: the kernel a step of `batch` rows runs."""
        r = self._lib.moe_decode_step_path(self.handle, int(batch))
        if r < 0:
            _check(r, "moe_decode_step_path")
        return r

    TRACE_FIELDS = ("start", "nready", "sched", "first_expert", "first_down", "prod_end", "mac_end",
                    "epi_end", "exit", "prod_wait_slot_cyc", "prod_wait_dep_cyc", "prod_grab_cyc",
                    "mac_wait_full_cyc", "mac_wait_rb_cyc", "epi_busy_cyc", "units",
                    "mac_compute_cyc", "mac_stages", "prod_issue_cyc", "prod_stages", "mac_sched_cyc",
                    "mac_reduce_cyc", "mac_loop_cyc", "prod_setup_cyc", "prod_sched_cyc",
                    "prod_loop_cyc", "router_seen", "sched_built", "topk_done", "topk_synced",
                    "unique_done", "n_published", "topk_loaded", "topk_selected", "topk_chosen",
                    "topk_cyc", "sched_placed", "sched_sorted", "start_clk", "r39", "roles",
                    "first_tma", "norm_summed", "norm_reduced", "norm_stored", "conv_wait_cyc", "conv_work_cyc",
                    "mma_wait_conv_cyc")

    def trace_slots(self) -> int:
        return self._lib.moe_decode_trace_slots(self.handle)

    def set_trace(self, buf) -> None:
        """buf: None, or a device uint64/int64 tensor of n_layers * trace_slots() values."""
        _check(self._lib.moe_decode_set_trace(self.handle, _ptr(buf)), "moe_decode_set_trace")

    def close(self) -> None:
        if getattr(self, "handle", None):
            self._lib.moe_decode_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
