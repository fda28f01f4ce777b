"""ctypes binding of the generator twin (libmoegen.so): fill device tensors or
host numpy arrays with exactly the values ``moe_inputs`` defines."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import weight_spec, h_tensor_id, TID_E, Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoegen.so")
_SRC = os.path.join(_HERE, "gen.cu")
_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(_SRC):
        return LIB_PATH
    cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-ffp-contract=off",
           "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-o", LIB_PATH, _SRC]
    subprocess.run(cmd, check=True)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            build()
        L = ctypes.CDLL(LIB_PATH)
        L.moe_gen_fill_device.restype = ctypes.c_int
        L.moe_gen_fill_device.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_void_p]
        L.moe_gen_fill_host.restype = None
        L.moe_gen_fill_host.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                        ctypes.c_double, ctypes.c_double, ctypes.c_int]
        L.moe_gen_stream_key.restype = ctypes.c_uint64
        L.moe_gen_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        _lib = L
    return _lib


def fill_device(ptr: int, count: int, bf16: bool, seed: int, tensor_id: int, start: int,
                sigma: float = 1.0, uniform=None, stream: int = 0) -> None:
    kind, p0, p1 = (0, float(sigma), 0.0) if uniform is None else \
        (1, float(uniform[0]), float(uniform[1]) - float(uniform[0]))
    rc = lib().moe_gen_fill_device(ctypes.c_void_p(ptr), count, int(bf16), kind, seed, tensor_id,
                                   start, p0, p1, ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"moe_gen_fill_device failed with CUDA error {rc}")


def fill_host(count: int, bf16: bool, seed: int, tensor_id: int, start: int, sigma: float = 1.0,
              uniform=None, threads: int = 0) -> np.ndarray:
    """Host twin: returns uint16 bf16 bits (bf16=True) or float32."""
    kind, p0, p1 = (0, float(sigma), 0.0) if uniform is None else \
        (1, float(uniform[0]), float(uniform[1]) - float(uniform[0]))
    out = np.empty(count, dtype=np.uint16 if bf16 else np.float32)
    lib().moe_gen_fill_host(out.ctypes.data_as(ctypes.c_void_p), count, int(bf16), kind, seed,
                            tensor_id, start, p0, p1, threads or (os.cpu_count() or 1))
    return out


def weight_host(w: Workload, which: str, expert: int, threads: int = 0) -> np.ndarray:
    """One expert's weight slice [rows, cols] as float32 (exact bf16 values for bf16
    workloads), generated on the host by the C twin (fast path of gen_weight)."""
    from . import bf16_bits_to_f32
    tid, n, rows, cols, sigma = weight_spec(w, which)
    per = rows * cols
    x = fill_host(per, w.dtype != "f32", w.seed, tid, expert * per, sigma, threads=threads)
    return (bf16_bits_to_f32(x) if w.dtype != "f32" else x).reshape(rows, cols)
