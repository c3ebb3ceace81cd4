"""Device-side fills that equal workload/gen.py bit for bit (libodagen.so, built in-tree).

Used to put large seeded inputs (the prefilled KV pools, per-step q/k/v) straight into HBM
without a host copy.  Holds no arithmetic of the method.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

from . import gen

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "lib", "libodagen.so")
SRC = os.path.join(HERE, "csrc", "gen.cu")
_lib = None
_tables = {}


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", SRC, "-o", LIB, "-lcudart_static", "-lrt", "-ldl",
           "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for the workload generator:\n" + r.stdout + r.stderr)
    return LIB


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing: run workload.device.build() first")
        L = ctypes.CDLL(LIB)
        L.odagen_fill_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                              ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
        L.odagen_fill_normal_bf16.restype = ctypes.c_int
        L.odagen_fill_kv.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                     ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        L.odagen_fill_kv.restype = ctypes.c_int
        _lib = L
    return _lib


def table(device, log2_scale: int = 0) -> torch.Tensor:
    device = torch.device(device)
    if (device, log2_scale) not in _tables:
        t = torch.from_numpy(gen.normal_bf16_table(log2_scale).view(np.int16)).to(device)
        _tables[(device, log2_scale)] = t
    return _tables[(device, log2_scale)]


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def fill_normal_bf16(out: torch.Tensor, key: int, start: int = 0, log2_scale: int = 0) -> torch.Tensor:
    """Fill a contiguous 2-byte tensor (bf16 or int16) with draws start.. of stream ``key``
    (N(0,1) times 2^log2_scale, as gen.normal_bf16)."""
    assert out.is_cuda and out.is_contiguous() and out.element_size() == 2
    rc = lib().odagen_fill_normal_bf16(ctypes.c_void_p(out.data_ptr()), out.numel(),
                                       ctypes.c_uint64(key & (2**64 - 1)), ctypes.c_uint64(start),
                                       ctypes.c_void_p(table(out.device, log2_scale).data_ptr()),
                                       _stream(out.device))
    if rc != 0:
        raise RuntimeError(f"odagen_fill_normal_bf16 failed: cudaError {rc}")
    return out


def fill_kv(pool: torch.Tensor, page_table: torch.Tensor, n_tokens, keys, Hkv: int) -> None:
    """Prefill a pool [n_pages, Hkv, 16, 128] (2-byte elements) for every sequence."""
    assert pool.is_cuda and pool.is_contiguous() and pool.element_size() == 2
    B, max_pages = page_table.shape
    dev = pool.device
    nt = torch.tensor(list(n_tokens), dtype=torch.int32, device=dev)
    ks = torch.tensor([k & (2**63 - 1) if k < 2**63 else k - 2**64 for k in keys],
                      dtype=torch.int64, device=dev)
    rc = lib().odagen_fill_kv(ctypes.c_void_p(pool.data_ptr()), ctypes.c_void_p(page_table.data_ptr()),
                              B, max_pages, Hkv, ctypes.c_void_p(nt.data_ptr()),
                              ctypes.c_void_p(ks.data_ptr()), int(max(n_tokens)),
                              int(pool.shape[0]), ctypes.c_void_p(table(dev).data_ptr()),
                              _stream(dev))
    if rc != 0:
        raise RuntimeError(f"odagen_fill_kv failed: cudaError {rc}")
    torch.cuda.current_stream(dev).synchronize()
