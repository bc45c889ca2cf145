"""Binding of rkv_compress_step_noalloc: the compression step for callers that
cannot allocate device memory (a plugin inside an engine that owns the whole
GPU, a decode loop where allocating is not allowed).  The library supplies the
step's scratch from a fixed array in its own device memory, so batch is limited
to RKV_NOALLOC_MAX_BATCH sequences and overlapping calls must be serialised.
Argument marshalling only, like the rest of the binding."""
from __future__ import annotations

import ctypes

import torch

from . import (_check, _dtype, _lib, _ptr, _ptr_array, _stream, rkv_config,  # noqa: F401
               rkv_step_options)

RKV_NOALLOC_MAX_BATCH = 4096

_f = _lib.rkv_compress_step_noalloc
_f.restype = ctypes.c_int
_f.argtypes = [ctypes.POINTER(rkv_config), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
               ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(rkv_step_options),
               ctypes.c_void_p]

_fs = _lib.rkv_noalloc_status
_fs.restype = ctypes.c_int
_fs.argtypes = [ctypes.c_void_p]


def rkv_noalloc_status(stream=None) -> int:
    """Device-side status of the latest allocation-free call on the current
    device (synchronises the stream): 0, or the RKV_STATUS_DEVICE_TIMEOUT /
    RKV_ERR_DEVICE_INPUT code."""
    return int(_fs(_stream(stream)))


def rkv_compress_step_noalloc(cfg, k_layers, v_layers, q_layers, cur_len, budgets=None,
                              lambdas=None, kept_out=None, scores_out=None, cluster_size=0,
                              stream=None):
    """Same arguments as rkv_compress_step, without a workspace."""
    k_layers, v_layers, q_layers = list(k_layers), list(v_layers), list(q_layers)
    batch, _, cap, _ = k_layers[0].shape
    for t in k_layers + v_layers + q_layers:
        _dtype(t, torch.bfloat16, "k/v/q")
    _dtype(cur_len, torch.int32, "cur_len"); _dtype(budgets, torch.int32, "budgets")
    _dtype(lambdas, torch.float32, "lambdas"); _dtype(kept_out, torch.int32, "kept_out")
    _dtype(scores_out, torch.float32, "scores_out")
    opts = rkv_step_options(_ptr(kept_out), _ptr(scores_out), None, None, int(cluster_size))
    return _check(_f(ctypes.byref(cfg), len(k_layers), batch, cap, _ptr_array(k_layers),
                     _ptr_array(v_layers), _ptr_array(q_layers), _ptr(budgets), _ptr(lambdas),
                     _ptr(cur_len), ctypes.byref(opts), _stream(stream)),
                  "rkv_compress_step_noalloc", allow_disabled=True)
