"""Seeded synthetic inputs for the MoE decode-layer workloads.

This package generates inputs only; it holds none of the layer's arithmetic.
It is the one module that both the CPU oracle side (tests, the timed CPU
baseline) and the GPU side (tests, bench) use, so that any expert's weights
can be regenerated on the host bit-identically to what the device holds.

The element generator is defined in ``moe_synth.h`` (SplitMix64 counter
stream, Irwin-Hall normal approximation, bf16 round-to-nearest-even).

Workloads (``WORKLOADS``) follow the five layer configurations the decode path
is measured on: a tiny CPU-sized layer, and the 7168-hidden / 896-expert /
top-16 layer at batch 1, batch 8, batch 64 with a Zipf-skewed router, and a
32-row two-layer speculative-verify shape.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libmoe_synth_host.so")
CUDA_LIB = os.path.join(_HERE, "libmoe_synth_cuda.so")

KIND_GAMMA = 1
KIND_W_ROUTER = 2
KIND_W_GATE = 3
KIND_W_UP = 4
KIND_W_DOWN = 5
KIND_WS_GATE = 6
KIND_WS_UP = 7
KIND_WS_DOWN = 8
KIND_X = 9
KIND_BIAS_PERM = 10
KIND_ROW_NOISE = 11
KIND_ROW_BASE = 12
KIND_WQ_GATE = 13   # FP8 expert weights: E4M3 codes
KIND_WQ_UP = 14
KIND_WQ_DOWN = 15
KIND_SQ_GATE = 16   # FP8 expert weights: per-block scale exponents
KIND_SQ_UP = 17
KIND_SQ_DOWN = 18
FP8_BLOCK = 128     # scale blocks are FP8_BLOCK x FP8_BLOCK elements


def tensor_id(layer: int, kind: int) -> int:
    return (int(layer) << 8) | int(kind)


def build(verbose: bool = False) -> None:
    """Compile the host fill library (gcc) and the device fill library (nvcc, sm_100a)."""
    cmds = [
        ["gcc", "-O3", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
         "-o", HOST_LIB, os.path.join(_HERE, "synth_host.c"), "-lm"],
        ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
         "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-o", CUDA_LIB, os.path.join(_HERE, "synth_cuda.cu")],
    ]
    for cmd in cmds:
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True, cwd=_HERE)


_host = None
_cuda = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            build()
        lib = ctypes.CDLL(HOST_LIB)
        u64, f32 = ctypes.c_uint64, ctypes.c_float
        vp = ctypes.c_void_p
        lib.ms_fill_host.argtypes = [u64, u64, u64, u64, f32, f32, vp]
        lib.ms_fill_host.restype = None
        lib.ms_z_host.argtypes = [u64, u64, u64, u64, vp]
        lib.ms_z_host.restype = None
        lib.ms_words_host.argtypes = [u64, u64, u64, u64, vp]
        lib.ms_words_host.restype = None
        lib.ms_mix64_host.argtypes = [u64]
        lib.ms_mix64_host.restype = u64
        lib.ms_fill_rows_correlated.argtypes = [u64, ctypes.c_uint32, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, vp]
        lib.ms_fill_rows_correlated.restype = None
        lib.ms_router_bias.argtypes = [u64, ctypes.c_uint32, ctypes.c_int, vp]
        lib.ms_router_bias.restype = None
        lib.ms_fill_e4m3_host.argtypes = [u64, u64, u64, u64, vp]
        lib.ms_fill_e4m3_host.restype = None
        lib.ms_e4m3_encode_host.argtypes = [vp, u64, vp]
        lib.ms_e4m3_encode_host.restype = None
        lib.ms_block_exps_host.argtypes = [u64, u64, u64, u64, ctypes.c_int, vp]
        lib.ms_block_exps_host.restype = None
        lib.ms_fill_e4m3_cover_host.argtypes = [u64, u64, u64, u64, u64, u64, ctypes.c_uint32, vp]
        lib.ms_fill_e4m3_cover_host.restype = None
        lib.ms_block_exps_cover_host.argtypes = [u64, u64, ctypes.c_uint32, ctypes.c_int, vp]
        lib.ms_block_exps_cover_host.restype = None
        _host = lib
    return _host


def _cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(CUDA_LIB):
            raise RuntimeError(f"{CUDA_LIB} is missing: run synth.build() first")
        lib = ctypes.CDLL(CUDA_LIB)
        u64, f32, vp = ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p
        lib.ms_fill_device.argtypes = [u64, u64, u64, u64, f32, f32, vp, vp]
        lib.ms_fill_device.restype = ctypes.c_int
        lib.ms_fill_e4m3_device.argtypes = [u64, u64, u64, u64, vp, vp]
        lib.ms_fill_e4m3_device.restype = ctypes.c_int
        lib.ms_fill_e4m3_cover_device.argtypes = [u64, u64, u64, u64, u64, u64, ctypes.c_uint32, vp, vp]
        lib.ms_fill_e4m3_cover_device.restype = ctypes.c_int
        _cuda = lib
    return _cuda


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def fill_host(seed: int, tid: int, start: int, n: int, sigma: float, mean: float = 0.0) -> np.ndarray:
    out = np.empty(int(n), dtype=np.uint16)
    _host_lib().ms_fill_host(seed, tid, start, n, np.float32(sigma), np.float32(mean), _ptr(out))
    return out


def z_host(seed: int, tid: int, start: int, n: int) -> np.ndarray:
    out = np.empty(int(n), dtype=np.float32)
    _host_lib().ms_z_host(seed, tid, start, n, _ptr(out))
    return out


def words_host(seed: int, tid: int, start: int, n: int) -> np.ndarray:
    out = np.empty(int(n), dtype=np.uint64)
    _host_lib().ms_words_host(seed, tid, start, n, _ptr(out))
    return out


def mix64(z: int) -> int:
    return int(_host_lib().ms_mix64_host(z))


def rows_correlated(seed: int, layer: int, nseq: int, rows_per_seq: int, H: int) -> np.ndarray:
    out = np.empty((nseq * rows_per_seq, H), dtype=np.uint16)
    _host_lib().ms_fill_rows_correlated(seed, layer, nseq, rows_per_seq, H, _ptr(out))
    return out


def router_bias(seed: int, layer: int, E: int) -> np.ndarray:
    out = np.empty(E, dtype=np.float32)
    _host_lib().ms_router_bias(seed, layer, E, _ptr(out))
    return out


def fill_e4m3_host(seed: int, tid: int, start: int, n: int) -> np.ndarray:
    """E4M3 codes (uint8) of elements start .. start + n - 1 of tensor tid."""
    out = np.empty(int(n), dtype=np.uint8)
    _host_lib().ms_fill_e4m3_host(seed, tid, start, n, _ptr(out))
    return out


def e4m3_encode_host(values) -> np.ndarray:
    """The generator's encoder: the E4M3 code nearest each fp32 value (ties to even),
    values clamped to [-448, 448]."""
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    out = np.empty(v.size, dtype=np.uint8)
    _host_lib().ms_e4m3_encode_host(_ptr(v), v.size, _ptr(out))
    return out


def block_exps_host(seed: int, tid: int, start: int, n: int, s0: int) -> np.ndarray:
    """Scale exponents (s0 - 1, s0 or s0 + 1) of blocks start .. start + n - 1."""
    out = np.empty(int(n), dtype=np.int32)
    _host_lib().ms_block_exps_host(seed, tid, start, n, int(s0), _ptr(out))
    return out


def fp8_s0(fan_in: int) -> int:
    """Central scale exponent of an FP8 matrix: 2^s0 * (448 / 6) is the power of two
    nearest 1/sqrt(fan_in), so the dequantised weights have about the bf16 weights'
    spread."""
    return int(np.round(np.log2((1.0 / np.sqrt(float(fan_in))) / (448.0 / 6.0))))


def fill_e4m3_device(ptr: int, seed: int, tid: int, start: int, n: int, stream: int = 0) -> None:
    rc = _cuda_lib().ms_fill_e4m3_device(seed, tid, start, n, ctypes.c_void_p(ptr), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"ms_fill_e4m3_device failed with cudaError {rc}")


# ---- coverage codes: every block's codes share one exponent field, cycling over all 16 ----
def cover_phase(seed: int) -> int:
    return int(seed) % 16


def cover_t(fan_in: int) -> int:
    """Coverage blocks' weights lie in [2^(t-3), 2^(t+1)): t = round(log2(1/sqrt(fan_in))) - 1."""
    return int(np.round(np.log2(1.0 / np.sqrt(float(fan_in))))) - 1


def fill_e4m3_cover_host(seed: int, tid: int, start: int, n: int, rows: int, cols: int) -> np.ndarray:
    """Coverage codes (uint8) of elements start .. start + n - 1 of a stack [E][rows][cols]."""
    out = np.empty(int(n), dtype=np.uint8)
    _host_lib().ms_fill_e4m3_cover_host(seed, tid, start, n, rows, cols, cover_phase(seed), _ptr(out))
    return out


def block_exps_cover_host(seed: int, start: int, n: int, fan_in: int) -> np.ndarray:
    out = np.empty(int(n), dtype=np.int32)
    _host_lib().ms_block_exps_cover_host(start, n, cover_phase(seed), cover_t(fan_in), _ptr(out))
    return out


def fill_e4m3_cover_device(ptr: int, seed: int, tid: int, start: int, n: int, rows: int, cols: int,
                           stream: int = 0) -> None:
    rc = _cuda_lib().ms_fill_e4m3_cover_device(seed, tid, start, n, rows, cols, cover_phase(seed),
                                               ctypes.c_void_p(ptr), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"ms_fill_e4m3_cover_device failed with cudaError {rc}")


def fill_device(ptr: int, seed: int, tid: int, start: int, n: int, sigma: float, mean: float = 0.0,
                stream: int = 0) -> None:
    rc = _cuda_lib().ms_fill_device(seed, tid, start, n, np.float32(sigma), np.float32(mean),
                                    ctypes.c_void_p(ptr), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"ms_fill_device failed with cudaError {rc}")


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (NaN -> quiet NaN)."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = ((u & 0x7F800000) == 0x7F800000) & ((u & 0x007FFFFF) != 0)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def sigma_for(fan_in: int) -> np.float32:
    """Weight standard deviation 1/sqrt(fan_in), rounded once to fp32."""
    return np.float32(1.0 / np.sqrt(float(fan_in)))


@dataclass(frozen=True)
class Workload:
    """One layer configuration and its seeded inputs."""

    name: str
    B: int
    H: int
    E: int
    k: int
    I: int
    Is: int
    seed: int
    layers: int = 1
    eps: float = 1e-6
    router: str = "uniform"        # "uniform" | "zipf"
    rows: str = "iid"              # "iid" | "correlated"
    nseq: int = 0
    rows_per_seq: int = 0
    gamma_sigma: float = 0.1
    # "bf16" | "fp8" (E4M3 codes with 128 x 128 block scales) | "fp8_cover" (FP8 with the
    # coverage codes: each block one exponent field, all 16 across the blocks)
    experts: str = "bf16"
    notes: str = field(default="", compare=False)

    # ---- hidden states --------------------------------------------------
    def x_host(self, batch: int | None = None) -> np.ndarray:
        """Input rows, bf16 bits [B, H] (layer 0 input)."""
        if self.rows == "correlated":
            x = rows_correlated(self.seed, 0, self.nseq, self.rows_per_seq, self.H)
        else:
            x = fill_host(self.seed, tensor_id(0, KIND_X), 0, self.B * self.H, 1.0).reshape(self.B, self.H)
        return x if batch is None else x[:batch].copy()

    def x_pool_host(self, count: int) -> np.ndarray:
        """`count` distinct input batches [count, B, H] for timing loops (variant v uses seed + 1000*v)."""
        out = np.empty((count, self.B, self.H), dtype=np.uint16)
        for v in range(count):
            s = self.seed + 1000 * v
            if self.rows == "correlated":
                out[v] = rows_correlated(s, 0, self.nseq, self.rows_per_seq, self.H)
            else:
                out[v] = fill_host(s, tensor_id(0, KIND_X), 0, self.B * self.H, 1.0).reshape(self.B, self.H)
        return out

    # ---- per-layer parameters --------------------------------------------
    def gamma_host(self, layer: int = 0) -> np.ndarray:
        return fill_host(self.seed, tensor_id(layer, KIND_GAMMA), 0, self.H, self.gamma_sigma, 1.0)

    def bias_host(self, layer: int = 0):
        if self.router != "zipf":
            return None
        return router_bias(self.seed, layer, self.E)

    def w_router_host(self, layer: int = 0) -> np.ndarray:
        return fill_host(self.seed, tensor_id(layer, KIND_W_ROUTER), 0, self.E * self.H,
                         sigma_for(self.H)).reshape(self.E, self.H)

    def shared_host(self, layer: int = 0):
        H, Is = self.H, self.Is
        g = fill_host(self.seed, tensor_id(layer, KIND_WS_GATE), 0, Is * H, sigma_for(H)).reshape(Is, H)
        u = fill_host(self.seed, tensor_id(layer, KIND_WS_UP), 0, Is * H, sigma_for(H)).reshape(Is, H)
        d = fill_host(self.seed, tensor_id(layer, KIND_WS_DOWN), 0, H * Is, sigma_for(Is)).reshape(H, Is)
        return g, u, d

    def expert_host(self, layer: int, e: int):
        """(W_gate[e] [I,H], W_up[e] [I,H], W_down[e] [H,I]) as bf16 bits."""
        H, I = self.H, self.I
        n = I * H
        g = fill_host(self.seed, tensor_id(layer, KIND_W_GATE), e * n, n, sigma_for(H)).reshape(I, H)
        u = fill_host(self.seed, tensor_id(layer, KIND_W_UP), e * n, n, sigma_for(H)).reshape(I, H)
        d = fill_host(self.seed, tensor_id(layer, KIND_W_DOWN), e * n, n, sigma_for(I)).reshape(H, I)
        return g, u, d

    # ---- device generation (whole tensors) ----------------------------------
    def device_specs(self, layer: int):
        """(name, kind, numel, sigma, mean) of every bf16 tensor of one layer."""
        H, E, I, Is = self.H, self.E, self.I, self.Is
        return [
            ("gamma", KIND_GAMMA, H, np.float32(self.gamma_sigma), 1.0),
            ("w_router", KIND_W_ROUTER, E * H, sigma_for(H), 0.0),
            ("w_gate", KIND_W_GATE, E * I * H, sigma_for(H), 0.0),
            ("w_up", KIND_W_UP, E * I * H, sigma_for(H), 0.0),
            ("w_down", KIND_W_DOWN, E * H * I, sigma_for(I), 0.0),
            ("ws_gate", KIND_WS_GATE, Is * H, sigma_for(H), 0.0),
            ("ws_up", KIND_WS_UP, Is * H, sigma_for(H), 0.0),
            ("ws_down", KIND_WS_DOWN, H * Is, sigma_for(Is), 0.0),
        ]

    def device_layer(self, layer: int, device="cuda", stream: int = 0) -> dict:
        """All of one layer's parameters generated on the device (torch tensors).

        bf16 tensors are returned as torch.bfloat16 holding exactly the bit
        patterns of the host generator; the router bias (zipf workloads) as fp32.
        """
        import torch

        out = {}
        for name, kind, numel, sigma, mean in self.device_specs(layer):
            t = torch.empty(int(numel), dtype=torch.bfloat16, device=device)
            fill_device(t.data_ptr(), self.seed, tensor_id(layer, kind), 0, int(numel), sigma, mean,
                        stream)
            out[name] = t
        H, E, I, Is = self.H, self.E, self.I, self.Is
        out["w_router"] = out["w_router"].view(E, H)
        out["w_gate"] = out["w_gate"].view(E, I, H)
        out["w_up"] = out["w_up"].view(E, I, H)
        out["w_down"] = out["w_down"].view(E, H, I)
        out["ws_gate"] = out["ws_gate"].view(Is, H)
        out["ws_up"] = out["ws_up"].view(Is, H)
        out["ws_down"] = out["ws_down"].view(H, Is)
        bias = self.bias_host(layer)
        out["router_bias"] = None if bias is None else torch.from_numpy(bias).to(device)
        return out

    # ---- FP8 expert weights (E4M3 codes, one power-of-two scale per 128 x 128 block) ----
    @property
    def is_fp8(self) -> bool:
        return self.experts in ("fp8", "fp8_cover")

    def fp8_matrices(self):
        """(name, code kind, scale kind, rows, cols, fan_in) of each expert matrix."""
        H, I = self.H, self.I
        return [("gate", KIND_WQ_GATE, KIND_SQ_GATE, I, H, H), ("up", KIND_WQ_UP, KIND_SQ_UP, I, H, H),
                ("down", KIND_WQ_DOWN, KIND_SQ_DOWN, H, I, I)]

    def fp8_scales_host(self, layer: int, which: str, experts=None) -> np.ndarray:
        """fp32 scales 2^exponent [len(experts)][rows/128][cols/128] of one matrix kind."""
        name, _, sk, rows, cols, fan_in = next(m for m in self.fp8_matrices() if m[0] == which)
        rb, cb = rows // FP8_BLOCK, cols // FP8_BLOCK
        experts = range(self.E) if experts is None else experts
        out = np.empty((len(experts), rb, cb), dtype=np.float32)
        for i, e in enumerate(experts):
            if self.experts == "fp8_cover":
                ex = block_exps_cover_host(self.seed, int(e) * rb * cb, rb * cb, fan_in)
            else:
                ex = block_exps_host(self.seed, tensor_id(layer, sk), int(e) * rb * cb, rb * cb, fp8_s0(fan_in))
            out[i] = np.ldexp(np.float32(1.0), ex).astype(np.float32).reshape(rb, cb)
        return out

    def expert_fp8_host(self, layer: int, e: int):
        """{gate, up, down: (E4M3 codes [rows, cols] uint8, fp32 block scales
        [rows/128, cols/128])} of expert e."""
        out = {}
        for name, qk, _, rows, cols, _ in self.fp8_matrices():
            if self.experts == "fp8_cover":
                codes = fill_e4m3_cover_host(self.seed, tensor_id(layer, qk), e * rows * cols, rows * cols, rows, cols)
            else:
                codes = fill_e4m3_host(self.seed, tensor_id(layer, qk), e * rows * cols, rows * cols)
            out[name] = (codes.reshape(rows, cols), self.fp8_scales_host(layer, name, [e])[0])
        return out

    def device_layer_fp8(self, layer: int, device="cuda", stream: int = 0) -> dict:
        """One layer with FP8 expert weights, generated on the device: gamma, router and
        shared expert bf16 as in device_layer; w_gate_q, w_up_q, w_down_q uint8 [E, rows,
        cols] and w_gate_scale, w_up_scale, w_down_scale fp32 [E, rows/128, cols/128]."""
        import torch

        out = {}
        for name, kind, numel, sigma, mean in self.device_specs(layer):
            if name in ("w_gate", "w_up", "w_down"):
                continue
            t = torch.empty(int(numel), dtype=torch.bfloat16, device=device)
            fill_device(t.data_ptr(), self.seed, tensor_id(layer, kind), 0, int(numel), sigma, mean, stream)
            out[name] = t
        H, E, Is = self.H, self.E, self.Is
        out["w_router"] = out["w_router"].view(E, H)
        out["ws_gate"] = out["ws_gate"].view(Is, H)
        out["ws_up"] = out["ws_up"].view(Is, H)
        out["ws_down"] = out["ws_down"].view(H, Is)
        for name, qk, _, rows, cols, _ in self.fp8_matrices():
            q = torch.empty((E, rows, cols), dtype=torch.uint8, device=device)
            if self.experts == "fp8_cover":
                fill_e4m3_cover_device(q.data_ptr(), self.seed, tensor_id(layer, qk), 0, E * rows * cols, rows, cols,
                                       stream)
            else:
                fill_e4m3_device(q.data_ptr(), self.seed, tensor_id(layer, qk), 0, E * rows * cols, stream)
            out[f"w_{name}_q"] = q
            out[f"w_{name}_scale"] = torch.from_numpy(self.fp8_scales_host(layer, name)).to(device)
        bias = self.bias_host(layer)
        out["router_bias"] = None if bias is None else torch.from_numpy(bias).to(device)
        return out

    def expert_bytes(self) -> int:
        """Bytes of one expert's weights as stored (codes and block scales when FP8)."""
        H, I = self.H, self.I
        if self.is_fp8:
            return 3 * I * H + 3 * (I // FP8_BLOCK) * (H // FP8_BLOCK) * 4
        return 3 * I * H * 2

    def device_layer_any(self, layer: int, device="cuda", stream: int = 0) -> dict:
        """device_layer, or device_layer_fp8 for a workload with FP8 experts."""
        if self.is_fp8:
            return self.device_layer_fp8(layer, device=device, stream=stream)
        return self.device_layer(layer, device=device, stream=stream)

    def weight_bytes_per_layer(self) -> int:
        return 2 * sum(s[2] for s in self.device_specs(0))


WORKLOADS = {
    0: Workload("tiny_b1_h256_e64_k4", B=1, H=256, E=64, k=4, I=128, Is=128, seed=0),
    1: Workload("b1_h7168_e896_k16", B=1, H=7168, E=896, k=16, I=1024, Is=2048, seed=1),
    2: Workload("b8_h7168_e896_k16", B=8, H=7168, E=896, k=16, I=1024, Is=2048, seed=2),
    3: Workload("b64_h7168_e896_k16_zipf", B=64, H=7168, E=896, k=16, I=1024, Is=2048, seed=3,
                router="zipf"),
    4: Workload("verify_4x8_h7168_e896_k16_2layer", B=32, H=7168, E=896, k=16, I=1024, Is=2048,
                seed=4, layers=2, rows="correlated", nseq=4, rows_per_seq=8),
}

# The same layers with FP8 expert weights (batch 1 and batch 8).
FP8_WORKLOADS = {
    1: Workload("b1_h7168_e896_k16_fp8", B=1, H=7168, E=896, k=16, I=1024, Is=2048, seed=1, experts="fp8"),
    2: Workload("b8_h7168_e896_k16_fp8", B=8, H=7168, E=896, k=16, I=1024, Is=2048, seed=2, experts="fp8"),
}
