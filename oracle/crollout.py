"""ctypes wrapper of ``rollout.c``: the plain sequential GRU evaluation on the
host in fp64 and fp32, OpenMP over the batch's independent sequences.

TEST AND BASELINE INFRASTRUCTURE ONLY (see the package docstring): it times
what a CPU does without the parallel Newton method, beside the GPU solve.  The
product path never loads it.  ``build()`` compiles the shared library in
place (gcc, -O3 for the x86-64-v3 level so that a library built on one host
runs on another, -fopenmp).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .cells import GRU

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "rollout.c")
LIB = os.path.join(HERE, "librollout.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile rollout.c into librollout.so next to it (if missing or older)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["gcc", "-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", SRC, "-o", LIB, "-lm"],
                       check=True)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        for name, real in (("gru_rollout_f64", ctypes.c_double), ("gru_rollout_f32", ctypes.c_float)):
            f = getattr(L, name)
            p = ctypes.POINTER(real)
            f.argtypes = [p, p, p, p, p, p] + [ctypes.c_int] * 5 + [p, ctypes.c_int]
            f.restype = ctypes.c_int
        for name, real in (("lstm_rollout_f64", ctypes.c_double), ("lstm_rollout_f32", ctypes.c_float)):
            f = getattr(L, name)
            p = ctypes.POINTER(real)
            f.argtypes = [p] * 7 + [ctypes.c_int] * 4 + [p, p, ctypes.c_int]
            f.restype = ctypes.c_int
        L.rollout_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().rollout_max_threads())


def rollout(cell: GRU, x: np.ndarray, h0: np.ndarray, dtype=np.float64, threads: int = 0) -> np.ndarray:
    """h [B, T, D] of the sequential evaluation, computed in `dtype` (float64
    or float32) from the cell's parameters and x [B, T, Din], h0 [B, D]."""
    dtype = np.dtype(dtype)
    real = ctypes.c_double if dtype == np.float64 else ctypes.c_float
    fn = lib().gru_rollout_f64 if dtype == np.float64 else lib().gru_rollout_f32
    arr = lambda a: np.ascontiguousarray(a, dtype=dtype)
    x_, wi, bi, wh, bh, h0_ = map(arr, (x, cell.w_ih, cell.b_ih, cell.w_hh, cell.b_hh, h0))
    B, T, din = x_.shape
    d = cell.d
    h = np.empty((B, T, d), dtype=dtype)
    ptr = lambda a: a.ctypes.data_as(ctypes.POINTER(real))
    rc = fn(ptr(x_), ptr(wi), ptr(bi), ptr(wh), ptr(bh), ptr(h0_), B, T, din, d,
            1 if cell.kind == "dense" else 0, ptr(h), int(threads))
    if rc != 0:
        raise RuntimeError("gru_rollout failed")
    return h


def lstm_rollout(cell, x: np.ndarray, c0: np.ndarray, h0: np.ndarray, dtype=np.float64, threads: int = 0):
    """(c, h) [B, T, D] of the diagonal LSTM's sequential evaluation in `dtype`
    (``cell``: oracle.lstm.LSTM)."""
    dtype = np.dtype(dtype)
    real = ctypes.c_double if dtype == np.float64 else ctypes.c_float
    fn = lib().lstm_rollout_f64 if dtype == np.float64 else lib().lstm_rollout_f32
    arr = lambda a: np.ascontiguousarray(a, dtype=dtype)
    x_, wi, bi, u, bh, c0_, h0_ = map(arr, (x, cell.w_ih, cell.b_ih, cell.u, cell.b_hh, c0, h0))
    B, T, din = x_.shape
    d = cell.d
    c = np.empty((B, T, d), dtype=dtype)
    h = np.empty((B, T, d), dtype=dtype)
    ptr = lambda a: a.ctypes.data_as(ctypes.POINTER(real))
    rc = fn(ptr(x_), ptr(wi), ptr(bi), ptr(u), ptr(bh), ptr(c0_), ptr(h0_), B, T, din, d, ptr(c), ptr(h),
            int(threads))
    if rc != 0:
        raise RuntimeError("lstm_rollout failed")
    return c, h
