"""Python binding of librkv.so, the B200 R-KV decode-time KV compression step.

Argument marshalling only: every function here turns torch tensors into raw
device pointers and calls the C-ABI function of the same name (declared in
``include/rkv.h``).  All computation runs in the library's CUDA kernels; there
is no CPU fallback, and importing this package fails if ``librkv.so`` has not
been built (``python -m decode_kv_cache_head_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "RKV_OK", "RKV_STATUS_DISABLED", "RKV_RED_MEAN", "RKV_RED_MAX", "RKV_GQA_MAX", "RKV_GQA_MEAN",
    "RkvError", "rkv_config", "rkv_step_options", "make_config", "library_path",
    "rkv_status_string", "rkv_version", "rkv_last_cuda_error", "rkv_workspace_size",
    "rkv_workspace_status",
    "rkv_query_step_shape",
    "rkv_score_importance", "rkv_score_redundancy", "rkv_select_topk", "rkv_compact_kv",
    "rkv_compress_step", "rkv_append_kv",
    "rkv_workspace_size_shared", "rkv_score_shared", "rkv_select_compact_shared",
    "rkv_paged_kv", "rkv_compress_step_paged",
    "rkv_ragged_kv", "rkv_compress_step_ragged", "ragged_rows",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "librkv.so")

RKV_OK = 0
RKV_STATUS_DISABLED = 1
RKV_RED_MEAN, RKV_RED_MAX = 0, 1
RKV_GQA_MAX, RKV_GQA_MEAN = 0, 1


class rkv_config(ctypes.Structure):
    _fields_ = [
        ("budget", ctypes.c_int32),
        ("buffer", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("mix_lambda", ctypes.c_float),
        ("redundancy_mode", ctypes.c_int32),
        ("gqa_pool", ctypes.c_int32),
    ]


class rkv_paged_kv(ctypes.Structure):
    _fields_ = [
        ("block_table", ctypes.c_void_p),
        ("max_blocks", ctypes.c_int32),
        ("page_rows", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("freed_pages", ctypes.c_void_p),
        ("n_freed", ctypes.c_void_p),
    ]


class rkv_ragged_kv(ctypes.Structure):
    _fields_ = [
        ("seq_row", ctypes.c_void_p),
        ("seq_cap", ctypes.c_void_p),
        ("pool_rows", ctypes.c_int64),
        ("max_cap", ctypes.c_int32),
    ]


class rkv_step_options(ctypes.Structure):
    _fields_ = [
        ("kept_out", ctypes.c_void_p),
        ("scores_out", ctypes.c_void_p),
        ("main_begin", ctypes.c_void_p),
        ("main_end", ctypes.c_void_p),
        ("cluster_size", ctypes.c_int32),
        ("sim_begin", ctypes.c_void_p),
        ("sim_end", ctypes.c_void_p),
    ]


def library_path() -> str:
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m decode_kv_cache_head_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    CFG = ctypes.POINTER(rkv_config)
    sig = {
        "rkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "rkv_version": (I32, []),
        "rkv_last_cuda_error": (I32, []),
        "rkv_workspace_size": (SZ, [CFG, I32, I32, I32]),
        "rkv_workspace_status": (ctypes.c_int, [P, P]),
        "rkv_query_step_shape": (ctypes.c_int, [CFG, I64, I32, ctypes.POINTER(I32),
                                                ctypes.POINTER(I32), ctypes.POINTER(SZ)]),
        "rkv_score_importance": (ctypes.c_int, [CFG, P, P, I64, I32, P, P, P, SZ, P]),
        "rkv_score_redundancy": (ctypes.c_int, [CFG, P, I64, I32, P, P, P, SZ, P]),
        "rkv_select_topk": (ctypes.c_int, [CFG, P, P, I32, P, P, P, SZ, P]),
        "rkv_compact_kv": (ctypes.c_int, [CFG, P, P, P, P, P, I64, I32, P, SZ, P]),
        "rkv_compress_step": (ctypes.c_int, [CFG, I32, I32, I32, P, P, P, P, P, P,
                                             ctypes.POINTER(rkv_step_options), P, SZ, P]),
        "rkv_append_kv": (ctypes.c_int, [CFG, I32, I32, I32, P, P, P, P, I32, P, P, SZ, P]),
        "rkv_workspace_size_shared": (SZ, [CFG, I32, I32, I32]),
        "rkv_compress_step_paged": (ctypes.c_int, [CFG, I32, I32, ctypes.POINTER(rkv_paged_kv), P,
                                                   P, P, P, P, P, ctypes.POINTER(rkv_step_options),
                                                   P, SZ, P]),
        "rkv_compress_step_ragged": (ctypes.c_int, [CFG, I32, I32, ctypes.POINTER(rkv_ragged_kv),
                                                    P, P, P, P, P, P,
                                                    ctypes.POINTER(rkv_step_options), P, SZ, P]),
        "rkv_score_shared": (ctypes.c_int, [CFG, I32, I32, I32, P, P, P, P, P, P, P, SZ, P]),
        "rkv_select_compact_shared": (ctypes.c_int, [CFG, I32, I32, I32, P, P, P, P, P, P, P, SZ,
                                                     P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


# Compile the library first when it is missing or older than its sources (the
# build module itself needs no library); without nvcc this raises.
from . import build as _build  # noqa: E402

_build.build()
_lib = _load()


class RkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == -7:   # RKV_ERR_CUDA: name the CUDA error behind it
            self.cuda_error = int(_lib.rkv_last_cuda_error())
            detail = f"; cudaError {self.cuda_error}"
        super().__init__(f"{where}: {rkv_status_string(status)} ({status}{detail})")


def rkv_status_string(status: int) -> str:
    return _lib.rkv_status_string(int(status)).decode()


def rkv_version() -> int:
    return int(_lib.rkv_version())


def rkv_last_cuda_error() -> int:
    return int(_lib.rkv_last_cuda_error())


def make_config(budget=1024, buffer=128, window=8, head_dim=128, n_kv_heads=8, n_q_heads=32,
                mix_lambda=0.1, redundancy_mode=RKV_RED_MEAN, gqa_pool=RKV_GQA_MAX) -> rkv_config:
    return rkv_config(int(budget), int(buffer), int(window), int(head_dim), int(n_kv_heads),
                      int(n_q_heads), float(mix_lambda), int(redundancy_mode), int(gqa_pool))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to librkv must be contiguous")
    return t.data_ptr()


def _dtype(t: Optional[torch.Tensor], dt: torch.dtype, name: str) -> None:
    if t is not None and t.dtype != dt:
        raise TypeError(f"{name} must be {dt}, got {t.dtype}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str, allow_disabled: bool = False) -> int:
    if status == RKV_OK or (allow_disabled and status == RKV_STATUS_DISABLED):
        return status
    raise RkvError(status, where)


def rkv_workspace_size(cfg: rkv_config, n_layers: int, batch: int, cap: int) -> int:
    return int(_lib.rkv_workspace_size(ctypes.byref(cfg), n_layers, batch, cap))


def rkv_query_step_shape(cfg: rkv_config, n_units: int, cap: int):
    """(cluster_size, rows_per_cta, smem_bytes) that rkv_compress_step uses for n_units
    units (layers x batch x KV heads) of `cap` rows; cluster_size 1 = one CTA per unit."""
    cs, rows, smem = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_size_t()
    _check(_lib.rkv_query_step_shape(ctypes.byref(cfg), int(n_units), int(cap), ctypes.byref(cs),
                                     ctypes.byref(rows), ctypes.byref(smem)),
           "rkv_query_step_shape")
    return cs.value, rows.value, smem.value


def rkv_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    return int(_lib.rkv_workspace_status(_ptr(workspace), _stream(stream)))


def rkv_score_importance(cfg, q, k, n_tokens, I, inv_norm=None, workspace=None, stream=None):
    """q [Hq, w, 128] bf16; k [Hkv, cap, 128] bf16; I [Hkv, N-w] fp32; inv_norm [Hkv, N] fp32."""
    _dtype(q, torch.bfloat16, "q"); _dtype(k, torch.bfloat16, "k")
    _dtype(I, torch.float32, "I"); _dtype(inv_norm, torch.float32, "inv_norm")
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(_lib.rkv_score_importance(ctypes.byref(cfg), _ptr(q), _ptr(k), k.shape[-2] * 128,
                                            int(n_tokens), _ptr(I), _ptr(inv_norm), _ptr(workspace),
                                            ws, _stream(stream)), "rkv_score_importance")


def rkv_score_redundancy(cfg, k, n_tokens, r=None, R=None, workspace=None, stream=None):
    """k [Hkv, cap, 128] bf16; r, R [Hkv, N-w] fp32."""
    _dtype(k, torch.bfloat16, "k"); _dtype(r, torch.float32, "r"); _dtype(R, torch.float32, "R")
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(_lib.rkv_score_redundancy(ctypes.byref(cfg), _ptr(k), k.shape[-2] * 128,
                                            int(n_tokens), _ptr(r), _ptr(R), _ptr(workspace), ws,
                                            _stream(stream)), "rkv_score_redundancy")


def rkv_select_topk(cfg, I, R, n_tokens, kept, Z=None, workspace=None, stream=None):
    """I, R [Hkv, N-w] fp32; kept [Hkv, budget] int32; Z [Hkv, N-w] fp32 or None."""
    _dtype(I, torch.float32, "I"); _dtype(R, torch.float32, "R")
    _dtype(kept, torch.int32, "kept"); _dtype(Z, torch.float32, "Z")
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(_lib.rkv_select_topk(ctypes.byref(cfg), _ptr(I), _ptr(R), int(n_tokens),
                                       _ptr(kept), _ptr(Z), _ptr(workspace), ws, _stream(stream)),
                  "rkv_select_topk", allow_disabled=True)


def rkv_compact_kv(cfg, k_src, v_src, kept, k_dst, v_dst, n_tokens, workspace=None, stream=None):
    """k/v [Hkv, cap, 128] bf16 (dst may be src: in place); kept [Hkv, budget] int32."""
    for n, t in (("k_src", k_src), ("v_src", v_src), ("k_dst", k_dst), ("v_dst", v_dst)):
        _dtype(t, torch.bfloat16, n)
    _dtype(kept, torch.int32, "kept")
    ws = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check(_lib.rkv_compact_kv(ctypes.byref(cfg), _ptr(k_src), _ptr(v_src), _ptr(kept),
                                      _ptr(k_dst), _ptr(v_dst), k_src.shape[-2] * 128,
                                      int(n_tokens), _ptr(workspace), ws, _stream(stream)),
                  "rkv_compact_kv", allow_disabled=True)


def _ptr_array(ts: Sequence[torch.Tensor]):
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = _ptr(t)
    return arr


def _layers(x, name: str):
    """Per-layer device pointers of bf16 tensors: (ctypes array, n_layers, the shape
    of one layer).  `x` is one contiguous [n_layers, ...] tensor, whose layer
    pointers follow from its stride without a view per layer, or a sequence of
    per-layer tensors."""
    if isinstance(x, torch.Tensor):
        _dtype(x, torch.bfloat16, name)
        if not x.is_contiguous():
            raise ValueError("tensors passed to librkv must be contiguous")
        n = int(x.shape[0])
        base, step = x.data_ptr(), x.stride(0) * x.element_size()
        return (ctypes.c_void_p * n)(*[base + i * step for i in range(n)]), n, tuple(x.shape[1:])
    ts = list(x)
    for t in ts:
        _dtype(t, torch.bfloat16, name)
    return _ptr_array(ts), len(ts), tuple(ts[0].shape)


def rkv_compress_step(cfg, k_layers, v_layers, q_layers, cur_len, workspace, budgets=None,
                      lambdas=None, kept_out=None, scores_out=None, events=None,
                      cluster_size=0, stream=None, sim_events=None):
    """The whole step over all layers of a batch, in place.

    k_layers / v_layers: sequences of [batch, Hkv, cap, 128] bf16 tensors (one
    per layer, or one [n_layers, batch, Hkv, cap, 128] tensor); q_layers:
    [batch, Hq, w, 128] per layer; cur_len [batch] int32 (updated);
    budgets [batch] int32 / lambdas [batch] fp32 or None; kept_out
    [n_layers, batch, Hkv, cap] int32 and scores_out [n_layers, batch, Hkv, 4,
    cap] fp32 optional; events: (begin, end) torch.cuda.Event recorded around
    the main kernel, or None; sim_events: the same around the similarity kernel
    (MAX redundancy).
    """
    kp, n_layers, (batch, _, cap, _) = _layers(k_layers, "k")
    vp, _, _ = _layers(v_layers, "v")
    qp, _, _ = _layers(q_layers, "q")
    _dtype(cur_len, torch.int32, "cur_len"); _dtype(budgets, torch.int32, "budgets")
    _dtype(lambdas, torch.float32, "lambdas"); _dtype(kept_out, torch.int32, "kept_out")
    _dtype(scores_out, torch.float32, "scores_out")
    opts = rkv_step_options(_ptr(kept_out), _ptr(scores_out), None, None, int(cluster_size))
    if events is not None:
        opts.main_begin = events[0].cuda_event
        opts.main_end = events[1].cuda_event
    if sim_events is not None:
        opts.sim_begin = sim_events[0].cuda_event
        opts.sim_end = sim_events[1].cuda_event
    ws = workspace.numel() * workspace.element_size()
    return _check(_lib.rkv_compress_step(ctypes.byref(cfg), n_layers, batch, cap,
                                         kp, vp, qp, _ptr(budgets), _ptr(lambdas),
                                         _ptr(cur_len), ctypes.byref(opts), _ptr(workspace), ws,
                                         _stream(stream)), "rkv_compress_step",
                  allow_disabled=True)


def rkv_append_kv(cfg, k_layers, v_layers, k_new_layers, v_new_layers, cur_len, workspace,
                  stream=None):
    """Appends [batch, Hkv, n_new, 128] rows per layer at cur_len, then cur_len += n_new."""
    kp, n_layers, (batch, _, cap, _) = _layers(k_layers, "k")
    vp, _, _ = _layers(v_layers, "v")
    knp, _, (_, _, n_new, _) = _layers(k_new_layers, "k_new")
    vnp, _, _ = _layers(v_new_layers, "v_new")
    _dtype(cur_len, torch.int32, "cur_len")
    ws = workspace.numel() * workspace.element_size()
    return _check(_lib.rkv_append_kv(ctypes.byref(cfg), n_layers, batch, cap,
                                     kp, vp, knp, vnp, n_new,
                                     _ptr(cur_len), _ptr(workspace), ws, _stream(stream)),
                  "rkv_append_kv")


def rkv_workspace_size_shared(cfg: rkv_config, n_layers: int, batch: int, cap: int) -> int:
    return int(_lib.rkv_workspace_size_shared(ctypes.byref(cfg), int(n_layers), int(batch),
                                              int(cap)))


def rkv_score_shared(cfg, k_layers, q_layers, cur_len, z_sum, workspace, budgets=None,
                     lambdas=None, stream=None):
    """Shared selection, part 1: z_sum [n_layers, batch, cap] fp32 = the sum over
    this call's KV heads of their joint scores (cur_len is only read)."""
    kp, n_layers, (batch, _, cap, _) = _layers(k_layers, "k")
    qp, _, _ = _layers(q_layers, "q")
    _dtype(cur_len, torch.int32, "cur_len"); _dtype(budgets, torch.int32, "budgets")
    _dtype(lambdas, torch.float32, "lambdas"); _dtype(z_sum, torch.float32, "z_sum")
    ws = workspace.numel() * workspace.element_size()
    return _check(_lib.rkv_score_shared(ctypes.byref(cfg), n_layers, batch, cap,
                                        kp, qp, _ptr(budgets),
                                        _ptr(lambdas), _ptr(cur_len), _ptr(z_sum),
                                        _ptr(workspace), ws, _stream(stream)),
                  "rkv_score_shared", allow_disabled=True)


def rkv_select_compact_shared(cfg, k_layers, v_layers, cur_len, z_sum, workspace, budgets=None,
                              kept_out=None, stream=None):
    """Shared selection, part 2 (after z_sum is complete over the ranks): one kept
    set per (layer, sequence), every head of this call compacted in place."""
    kp, n_layers, (batch, _, cap, _) = _layers(k_layers, "k")
    vp, _, _ = _layers(v_layers, "v")
    _dtype(cur_len, torch.int32, "cur_len"); _dtype(budgets, torch.int32, "budgets")
    _dtype(z_sum, torch.float32, "z_sum"); _dtype(kept_out, torch.int32, "kept_out")
    ws = workspace.numel() * workspace.element_size()
    return _check(_lib.rkv_select_compact_shared(ctypes.byref(cfg), n_layers, batch, cap,
                                                 kp, vp,
                                                 _ptr(budgets), _ptr(cur_len), _ptr(z_sum),
                                                 _ptr(kept_out), _ptr(workspace), ws,
                                                 _stream(stream)),
                  "rkv_select_compact_shared", allow_disabled=True)


def rkv_compress_step_paged(cfg, k_pools, v_pools, q_layers, cur_len, workspace, block_table,
                            page_rows, freed_pages, n_freed, budgets=None, lambdas=None,
                            kept_out=None, scores_out=None, events=None, stream=None):
    """The step on paged caches, in place.

    k_pools / v_pools: per layer [num_pages, Hkv, page_rows, 128] bf16 (or one
    [n_layers, ...] tensor); block_table [batch, max_blocks] int32 (logical page
    j of sequence b); freed_pages [batch, max_blocks] / n_freed [batch] int32
    receive the pages each compressed sequence gives back.  kept_out /
    scores_out as in rkv_compress_step with cap = max_blocks * page_rows.
    """
    kp, n_layers, (num_pages, _, _, _) = _layers(k_pools, "k")
    vp, _, _ = _layers(v_pools, "v")
    qp, _, _ = _layers(q_layers, "q")
    batch, max_blocks = block_table.shape
    for t, n in ((cur_len, "cur_len"), (budgets, "budgets"), (block_table, "block_table"),
                 (freed_pages, "freed_pages"), (n_freed, "n_freed"), (kept_out, "kept_out")):
        _dtype(t, torch.int32, n)
    _dtype(lambdas, torch.float32, "lambdas"); _dtype(scores_out, torch.float32, "scores_out")
    pg = rkv_paged_kv(_ptr(block_table), int(max_blocks), int(page_rows), int(num_pages),
                      _ptr(freed_pages), _ptr(n_freed))
    opts = rkv_step_options(_ptr(kept_out), _ptr(scores_out), None, None, 0)
    if events is not None:
        opts.main_begin = events[0].cuda_event
        opts.main_end = events[1].cuda_event
    ws = workspace.numel() * workspace.element_size()
    return _check(_lib.rkv_compress_step_paged(ctypes.byref(cfg), n_layers, batch,
                                               ctypes.byref(pg), kp, vp, qp,
                                               _ptr(budgets), _ptr(lambdas), _ptr(cur_len),
                                               ctypes.byref(opts), _ptr(workspace), ws,
                                               _stream(stream)),
                  "rkv_compress_step_paged", allow_disabled=True)


def ragged_rows(caps, n_kv_heads: int):
    """First pool row of every sequence when the blocks [n_kv_heads][cap_b][128]
    are packed back to back in batch order, and the pool's row count."""
    rows, r = [], 0
    for c in caps:
        rows.append(r)
        r += int(n_kv_heads) * int(c)
    return rows, r


def rkv_compress_step_ragged(cfg, k_pools, v_pools, q_layers, cur_len, workspace, seq_row,
                             seq_cap, max_cap, budgets=None, lambdas=None, kept_out=None,
                             scores_out=None, events=None, sim_events=None, cluster_size=0,
                             stream=None):
    """The step on caches with per-sequence capacities, in place.

    k_pools / v_pools: per layer [pool_rows, 128] bf16 (or one [n_layers,
    pool_rows, 128] tensor); sequence b's [Hkv][seq_cap[b]][128] block starts at
    pool row seq_row[b] (seq_row [batch] int64, seq_cap [batch] int32, on the
    device); max_cap >= every seq_cap.  q_layers, cur_len, budgets, lambdas as in
    rkv_compress_step; kept_out [n_layers, batch, Hkv, max_cap] int32 and
    scores_out [n_layers, batch, Hkv, 4, max_cap] fp32 optional.
    """
    kp, n_layers, (pool_rows, _) = _layers(k_pools, "k")
    vp, _, _ = _layers(v_pools, "v")
    qp, _, (batch, _, _, _) = _layers(q_layers, "q")
    _dtype(seq_row, torch.int64, "seq_row"); _dtype(seq_cap, torch.int32, "seq_cap")
    _dtype(cur_len, torch.int32, "cur_len"); _dtype(budgets, torch.int32, "budgets")
    _dtype(lambdas, torch.float32, "lambdas"); _dtype(kept_out, torch.int32, "kept_out")
    _dtype(scores_out, torch.float32, "scores_out")
    rg = rkv_ragged_kv(_ptr(seq_row), _ptr(seq_cap), int(pool_rows), int(max_cap))
    opts = rkv_step_options(_ptr(kept_out), _ptr(scores_out), None, None, int(cluster_size))
    if events is not None:
        opts.main_begin = events[0].cuda_event
        opts.main_end = events[1].cuda_event
    if sim_events is not None:
        opts.sim_begin = sim_events[0].cuda_event
        opts.sim_end = sim_events[1].cuda_event
    ws = workspace.numel() * workspace.element_size()
    return _check(_lib.rkv_compress_step_ragged(ctypes.byref(cfg), n_layers, int(batch),
                                                ctypes.byref(rg), kp, vp, qp, _ptr(budgets),
                                                _ptr(lambdas), _ptr(cur_len), ctypes.byref(opts),
                                                _ptr(workspace), ws, _stream(stream)),
                  "rkv_compress_step_ragged", allow_disabled=True)
