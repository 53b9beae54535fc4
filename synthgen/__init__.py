"""Seeded synthetic-input generator (test and benchmark infrastructure).

Produces every random input the tests and the benchmark use -- fp32/fp16
tensors, token ids and block-quantized weight matrices -- as a pure function of
(seed, tensor name, element index).  The host library (``libsynthgen.so``) and
its CUDA twin (``libsynthgen_cuda.so``) emit identical bytes; the oracle and the
CUDA path both consume them, and neither imports the other.

Tensor streams are keyed by ``(seed, fnv1a(name))``.  Workload seeds are
``SEED_BASE + workload number``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libsynthgen.so")
CUDA_SO = os.path.join(HERE, "libsynthgen_cuda.so")

SEED_BASE = 0x4E54580

F32, F16, Q4_0, Q8_0, Q4_K, Q5_K, Q6_K = 0, 1, 2, 8, 12, 13, 14
BLOCK_ELEMS = {F32: 1, F16: 1, Q4_0: 32, Q8_0: 32, Q4_K: 256, Q5_K: 256, Q6_K: 256}
BLOCK_BYTES = {F32: 4, F16: 2, Q4_0: 18, Q8_0: 34, Q4_K: 144, Q5_K: 176, Q6_K: 210}

_NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build(force: bool = False) -> None:
    """Compile the host library (gcc) and the CUDA twin (nvcc, sm_100a)."""
    src = os.path.join(HERE, "synthgen.c")
    hdr = os.path.join(HERE, "sg_core.h")
    newest = max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not os.path.exists(HOST_SO) or os.path.getmtime(HOST_SO) < newest:
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
                               "-o", HOST_SO, src])
    csrc = os.path.join(HERE, "synthgen_cuda.cu")
    newest = max(os.path.getmtime(csrc), os.path.getmtime(hdr))
    if force or not os.path.exists(CUDA_SO) or os.path.getmtime(CUDA_SO) < newest:
        subprocess.check_call([_NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-Xcompiler", "-fPIC", "-shared", "-o", CUDA_SO, csrc])


_host = None
_cuda = None


def host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_SO):
            build()
        L = ctypes.CDLL(HOST_SO)
        i64, u32, u64, dbl, vp = ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
        L.sg_tensor_id.argtypes = [ctypes.c_char_p]
        L.sg_tensor_id.restype = u32
        L.sg_philox.argtypes = [vp, vp, vp]
        L.sg_normal_at.argtypes = [u32, u32, u64]
        L.sg_normal_at.restype = dbl
        L.sg_ln.argtypes = [dbl]
        L.sg_ln.restype = dbl
        L.sg_half_from_float.argtypes = [ctypes.c_float]
        L.sg_half_from_float.restype = ctypes.c_uint16
        L.sg_half_to_float.argtypes = [ctypes.c_uint16]
        L.sg_half_to_float.restype = ctypes.c_float
        L.sg_fill_f32.argtypes = [u32, u32, i64, dbl, dbl, vp, ctypes.c_int]
        L.sg_fill_f16.argtypes = [u32, u32, i64, dbl, dbl, vp, ctypes.c_int]
        L.sg_quant_rows.argtypes = [ctypes.c_int, u32, u32, i64, i64, i64, dbl, dbl, vp, ctypes.c_int]
        L.sg_quant_rows.restype = ctypes.c_int
        L.sg_quantize.argtypes = [ctypes.c_int, vp, i64, vp]
        L.sg_quantize.restype = ctypes.c_int
        L.sg_fill_tokens.argtypes = [u32, u32, i64, u32, vp]
        _host = L
    return _host


def cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(CUDA_SO):
            build()
        L = ctypes.CDLL(CUDA_SO)
        i64, u32, dbl, vp = ctypes.c_int64, ctypes.c_uint32, ctypes.c_double, ctypes.c_void_p
        L.sgc_fill_f32.argtypes = [u32, u32, i64, dbl, dbl, vp, vp]
        L.sgc_fill_f16.argtypes = [u32, u32, i64, dbl, dbl, vp, vp]
        L.sgc_fill_tokens.argtypes = [u32, u32, i64, u32, vp, vp]
        L.sgc_quant_rows.argtypes = [ctypes.c_int, u32, u32, i64, i64, i64, dbl, dbl, vp, vp]
        for f in (L.sgc_fill_f32, L.sgc_fill_f16, L.sgc_fill_tokens, L.sgc_quant_rows):
            f.restype = ctypes.c_int
        _cuda = L
    return _cuda


def _threads(n):
    return n if n else min(32, os.cpu_count() or 1)


def tensor_id(name: str) -> int:
    return int(host_lib().sg_tensor_id(name.encode()))


def row_bytes(qtype: int, K: int) -> int:
    return K // BLOCK_ELEMS[qtype] * BLOCK_BYTES[qtype]


# ------------------------------------------------------------------ host side
def philox(ctr, key):
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    host_lib().sg_philox(c, k, o)
    return list(o)


def normal_at(seed: int, name: str, idx: int) -> float:
    return host_lib().sg_normal_at(seed, tensor_id(name), idx)


def fill_f32(seed: int, name: str, n: int, mean: float = 0.0, sigma: float = 1.0, nthreads: int | None = None):
    out = np.empty(n, dtype=np.float32)
    host_lib().sg_fill_f32(seed, tensor_id(name), n, mean, sigma, out.ctypes.data, _threads(nthreads))
    return out


def fill_f16(seed: int, name: str, n: int, mean: float = 0.0, sigma: float = 1.0, nthreads: int | None = None):
    """fp16 bit patterns (uint16)."""
    out = np.empty(n, dtype=np.uint16)
    host_lib().sg_fill_f16(seed, tensor_id(name), n, mean, sigma, out.ctypes.data, _threads(nthreads))
    return out


def quant_rows(qtype: int, seed: int, name: str, M: int, K: int, mean: float = 0.0, sigma: float = 0.02,
               row0: int = 0, nrows: int | None = None, nthreads: int | None = None):
    """Rows [row0, row0+nrows) of the quantized M x K matrix, uint8 [nrows, row_bytes]."""
    if nrows is None:
        nrows = M - row0
    out = np.empty((nrows, row_bytes(qtype, K)), dtype=np.uint8)
    rc = host_lib().sg_quant_rows(qtype, seed, tensor_id(name), row0, nrows, K, mean, sigma, out.ctypes.data,
                                  _threads(nthreads))
    if rc != 0:
        raise ValueError(f"sg_quant_rows: bad qtype/K ({qtype}, {K})")
    return out


def quantize(qtype: int, w) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.float32).ravel()
    nb = w.size // BLOCK_ELEMS[qtype]
    out = np.empty(nb * BLOCK_BYTES[qtype], dtype=np.uint8)
    if host_lib().sg_quantize(qtype, w.ctypes.data, w.size, out.ctypes.data) != 0:
        raise ValueError("sg_quantize: size not a multiple of the block")
    return out


def tokens(seed: int, name: str, n: int, V: int):
    out = np.empty(n, dtype=np.int32)
    host_lib().sg_fill_tokens(seed, tensor_id(name), n, V, out.ctypes.data)
    return out


def half_from_float(f: float) -> int:
    return int(host_lib().sg_half_from_float(f))


# ---------------------------------------------------------------- device twin
def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with {rc}")


def dev_fill_f32(seed, name, n, mean, sigma, ptr, stream=0):
    _check(cuda_lib().sgc_fill_f32(seed, tensor_id(name), n, mean, sigma, ptr, stream), "sgc_fill_f32")


def dev_fill_f16(seed, name, n, mean, sigma, ptr, stream=0):
    _check(cuda_lib().sgc_fill_f16(seed, tensor_id(name), n, mean, sigma, ptr, stream), "sgc_fill_f16")


def dev_tokens(seed, name, n, V, ptr, stream=0):
    _check(cuda_lib().sgc_fill_tokens(seed, tensor_id(name), n, V, ptr, stream), "sgc_fill_tokens")


def dev_quant_rows(qtype, seed, name, M, K, ptr, mean=0.0, sigma=0.02, row0=0, nrows=None, stream=0):
    if nrows is None:
        nrows = M - row0
    _check(cuda_lib().sgc_quant_rows(qtype, seed, tensor_id(name), row0, nrows, K, mean, sigma, ptr, stream),
           "sgc_quant_rows")
