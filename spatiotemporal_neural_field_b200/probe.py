"""Thin ctypes binding of ``libspin4d_probe.so`` (``include/spin4d_probe.h``):
the measurement probes behind the rooflines and the bounded-wait self-test.

These are bench and test tools beside the decoder, not part of it.  Argument
marshalling only; the import fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .spin4d import Spin4dError, _check, _ptr, _stream, c_i32, c_i64, c_u32, c_vp

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspin4d_probe.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError("libspin4d_probe.so is not built (run `python -m spatiotemporal_neural_field_b200.build`)")
lib = ctypes.CDLL(_LIB_PATH)

_SIGS = {
    "spin4d_probe_gather": (c_i32, [c_vp, ctypes.c_uint64, c_i32, c_i64, c_i32, c_u32, c_vp, c_vp]),
    "spin4d_probe_stream": (c_i32, [c_vp, ctypes.c_uint64, c_i32, c_i32, c_vp, c_vp]),
    "spin4d_probe_atomic": (c_i32, [c_vp, ctypes.c_uint64, c_i32, c_i64, c_i32, c_u32, c_vp]),
    "spin4d_probe_bulk_reduce": (c_i32, [c_vp, ctypes.c_uint64, c_i32, c_i64, c_i32, c_u32, c_vp]),
    "spin4d_probe_fma": (c_i32, [c_i64, c_i32, c_vp, c_vp]),
    "spin4d_selftest_wait_timeout": (c_i32, [c_u32, c_vp]),
    "spin4d_probe_check_device_errors": (c_i32, [c_i32]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)
__all__ = ["Spin4dError", "probe_gather", "probe_stream", "probe_atomic", "probe_bulk_reduce", "probe_fma",
           "selftest_wait_timeout", "check_device_errors"]


def probe_gather(buf: torch.Tensor, width: int, loads_per_thread: int, blocks: int, seed: int = 1,
                 sink: Optional[torch.Tensor] = None, stream=None) -> int:
    """Launches the random-gather probe; returns the number of `width`-byte
    units read (sectors for width 4/16, 128-byte lines for width 128)."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
    _check("spin4d_probe_gather", lib.spin4d_probe_gather(_ptr(buf), buf.numel() * buf.element_size(), width,
                                                          loads_per_thread, blocks, seed, _ptr(sink),
                                                          _stream(stream)))
    return blocks * 256 * loads_per_thread // (8 if width == 128 else 1)


def probe_atomic(buf: torch.Tensor, width: int, ops_per_thread: int, blocks: int, seed: int = 1, stream=None) -> int:
    """Random fp32 reductions of `width` bytes into `buf`; returns the count."""
    _check("spin4d_probe_atomic", lib.spin4d_probe_atomic(_ptr(buf), buf.numel() * buf.element_size(), width,
                                                          ops_per_thread, blocks, seed, _stream(stream)))
    return blocks * 256 * ops_per_thread


def probe_bulk_reduce(buf: torch.Tensor, rows_per_thread: int, blocks: int, seed: int = 1, row_bytes: int = 128,
                      stream=None) -> int:
    """Random bulk fp32 row reductions into `buf`; returns the rows added."""
    _check("spin4d_probe_bulk_reduce", lib.spin4d_probe_bulk_reduce(_ptr(buf), buf.numel() * buf.element_size(),
                                                                    row_bytes, rows_per_thread, blocks, seed,
                                                                    _stream(stream)))
    return blocks * 128 * rows_per_thread


def probe_stream(buf: torch.Tensor, passes: int, blocks: int, sink: Optional[torch.Tensor] = None,
                 stream=None) -> int:
    """Sequential-read probe; returns the bytes read."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
    nbytes = buf.numel() * buf.element_size()
    _check("spin4d_probe_stream", lib.spin4d_probe_stream(_ptr(buf), nbytes, passes, blocks, _ptr(sink),
                                                          _stream(stream)))
    return passes * nbytes


def probe_fma(iters: int, blocks: int, device, sink: Optional[torch.Tensor] = None, stream=None) -> int:
    """fp32 FMA-chain probe; returns the FLOPs executed."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int32, device=device)
    _check("spin4d_probe_fma", lib.spin4d_probe_fma(iters, blocks, _ptr(sink), _stream(stream)))
    return 16 * iters * blocks * 256


def selftest_wait_timeout(max_iters: int = 4096, stream=None) -> None:
    """Launches a kernel whose bounded wait must run out (failure-detection test)."""
    _check("spin4d_selftest_wait_timeout", lib.spin4d_selftest_wait_timeout(max_iters, _stream(stream)))


def check_device_errors(clear: bool = True) -> None:
    """Synchronous: raises if a bounded wait of this library ran out."""
    _check("spin4d_probe_check_device_errors", lib.spin4d_probe_check_device_errors(1 if clear else 0))
