"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This package generates inputs only: weights, cached K/V, hidden states, token
ids and batch shapes. It holds none of the serving iteration's arithmetic.
Values come from one counter-based specification (see ``synth_cpu.c``):
Philox4x32-10 keyed by (seed, tensor id), an Irwin-Hall normal of eight 16-bit
uniforms, one fp32 multiply, one fp32 add and a bf16 round to nearest even.
``synth_cpu.c`` (host, used by the oracle) and ``synth_gpu.cu`` (device, used to
fill large buffers in HBM) implement it separately; tests check them bitwise.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_CPU_SO = os.path.join(_HERE, "libnfsynth_cpu.so")
_GPU_SO = os.path.join(_HERE, "libnfsynth_gpu.so")

# Seeds of the input families.
SEED_WEIGHTS = 0
SEED_KV = 1
SEED_INPUTS = 2
SEED_BATCH = 3

# Tensor ids within SEED_WEIGHTS: (layer << 8) | kind.
W_Q, W_K, W_V, W_O, W_GATE, W_UP, W_DOWN, W_ATTN_NORM, W_FFN_NORM, W_ROUTER, W_ROUTER_BIAS = range(11)
W_EXPERT_BASE = 16  # expert e: 16 + 3e + {0 gate, 1 up, 2 down}
GLOBAL_LAYER = 0xFFFF
G_EMBED, G_LM_HEAD, G_FINAL_NORM = range(3)

# Tensor ids within SEED_INPUTS / SEED_BATCH.
IN_HIDDEN, IN_TOKENS = 0, 1
B_CTX_UNIFORM, B_PAGE_PERM, B_CTX_LOGNORMAL = 0, 1, 2


def weight_tid(layer: int, kind: int) -> int:
    return ((layer & 0xFFFF) << 8) | kind


def expert_kind(e: int, which: int) -> int:
    return W_EXPERT_BASE + 3 * e + which


def build_cpu(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth_cpu.c")
    if force or not os.path.exists(_CPU_SO) or os.path.getmtime(_CPU_SO) < os.path.getmtime(src):
        subprocess.check_call(
            ["gcc", "-O3", "-march=x86-64-v2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
             "-fPIC", "-shared", "-o", _CPU_SO, src]
        )
    return _CPU_SO


def build_gpu(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth_gpu.cu")
    if force or not os.path.exists(_GPU_SO) or os.path.getmtime(_GPU_SO) < os.path.getmtime(src):
        subprocess.check_call(
            ["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-fmad=false",
             "-Xcompiler", "-fPIC", "-shared", "-o", _GPU_SO, src]
        )
    return _GPU_SO


_cpu = None
_gpu = None


def _lib():
    global _cpu
    if _cpu is None:
        _cpu = ctypes.CDLL(build_cpu())
        u32, u64, i64, f32, vp = (ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int64,
                                  ctypes.c_float, ctypes.c_void_p)
        _cpu.nfs_philox4x32_10.argtypes = [vp, vp, vp]
        _cpu.nfs_fill_normal_bf16.argtypes = [u32, u32, u64, u64, f32, f32, vp]
        _cpu.nfs_gather_normal_bf16.argtypes = [u32, u32, vp, u64, f32, f32, vp]
        _cpu.nfs_fill_normal_bf16_ranges.argtypes = [u32, u32, vp, u64, u64, f32, f32, vp]
        _cpu.nfs_fill_normal_f32.argtypes = [u32, u32, u64, u64, f32, f32, vp]
        _cpu.nfs_fill_uniform_int.argtypes = [u32, u32, u64, u64, i64, i64, vp]
        _cpu.nfs_fill_raw.argtypes = [u32, u32, u64, u64, vp]
    return _cpu


def _gpulib():
    global _gpu
    if _gpu is None:
        _gpu = ctypes.CDLL(build_gpu())
        _gpu.nfs_gpu_fill_normal_bf16.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64,
                                                  ctypes.c_uint64, ctypes.c_float, ctypes.c_float,
                                                  ctypes.c_void_p, ctypes.c_void_p]
        _gpu.nfs_gpu_fill_normal_bf16.restype = ctypes.c_int
    return _gpu


def normal_scale(sigma: float) -> np.float32:
    """fp32 scale that maps the centred Irwin-Hall sum to standard deviation ``sigma``."""
    return np.float32(sigma / math.sqrt(8.0 * (65536.0 * 65536.0 - 1.0) / 12.0))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def philox(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    _lib().nfs_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def raw_words(seed: int, tid: int, offset: int, n: int) -> np.ndarray:
    out = np.zeros((n, 4), dtype=np.uint32)
    _lib().nfs_fill_raw(seed, tid, offset, n, _ptr(out))
    return out


def normal_bf16(seed: int, tid: int, n: int, sigma: float = 1.0, mean: float = 0.0,
                offset: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements [offset, offset + n)."""
    out = np.empty(int(n), dtype=np.uint16)
    _lib().nfs_fill_normal_bf16(seed, tid, offset, int(n), float(normal_scale(sigma)), float(np.float32(mean)),
                                _ptr(out))
    return out


def gather_normal_bf16(seed: int, tid: int, idx: np.ndarray, sigma: float = 1.0, mean: float = 0.0) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    out = np.empty(idx.shape, dtype=np.uint16)
    _lib().nfs_gather_normal_bf16(seed, tid, _ptr(idx), idx.size, float(normal_scale(sigma)),
                                  float(np.float32(mean)), _ptr(out))
    return out


def ranges_normal_bf16(seed: int, tid: int, starts: np.ndarray, length: int, sigma: float = 1.0,
                       mean: float = 0.0) -> np.ndarray:
    starts = np.ascontiguousarray(starts, dtype=np.uint64)
    out = np.empty((starts.size, int(length)), dtype=np.uint16)
    _lib().nfs_fill_normal_bf16_ranges(seed, tid, _ptr(starts), starts.size, int(length),
                                       float(normal_scale(sigma)), float(np.float32(mean)), _ptr(out))
    return out


def normal_f32(seed: int, tid: int, n: int, sigma: float = 1.0, mean: float = 0.0, offset: int = 0) -> np.ndarray:
    out = np.empty(int(n), dtype=np.float32)
    _lib().nfs_fill_normal_f32(seed, tid, offset, int(n), float(normal_scale(sigma)), float(np.float32(mean)),
                               _ptr(out))
    return out


def uniform_int(seed: int, tid: int, n: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    out = np.empty(int(n), dtype=np.int64)
    _lib().nfs_fill_uniform_int(seed, tid, offset, int(n), int(lo), int(hi), _ptr(out))
    return out


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    return bf16_to_f32(u16).astype(np.float64)


def gpu_fill_normal_bf16(ptr: int, n: int, seed: int, tid: int, sigma: float = 1.0, mean: float = 0.0,
                         offset: int = 0, stream: int = 0) -> None:
    """Fill ``n`` bf16 elements at device address ``ptr`` with elements [offset, offset+n)."""
    rc = _gpulib().nfs_gpu_fill_normal_bf16(seed, tid, offset, int(n), float(normal_scale(sigma)),
                                            float(np.float32(mean)), ctypes.c_void_p(ptr), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"nfs_gpu_fill_normal_bf16 failed with CUDA error {rc}")
