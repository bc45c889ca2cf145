"""The C-ABI library without a GPU: it builds, loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

from decode_kv_cache_head_b200 import build as rkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
rkv_build.build()

import decode_kv_cache_head_b200 as rkv  # noqa: E402

HEADER = os.path.join(ROOT, "include", "rkv.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rkv_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("rkv_score_importance", "rkv_score_redundancy", "rkv_select_topk",
              "rkv_compact_kv", "rkv_compress_step", "rkv_workspace_size",
              "rkv_workspace_status", "rkv_status_string", "rkv_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", rkv.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    lib = ctypes.CDLL(rkv.library_path())
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)
    # nothing but the C ABI is exported
    assert not [s for s in exported if s.startswith("_Z")]


def test_status_strings_and_version():
    assert rkv.rkv_status_string(0) == "RKV_OK"
    assert "DISABLED" in rkv.rkv_status_string(1)
    assert "WORKSPACE" in rkv.rkv_status_string(-5)
    assert rkv.rkv_version() >= 10000


def test_workspace_size():
    c = rkv.make_config()
    base = rkv.rkv_workspace_size(c, 32, 1, 1152)
    assert base >= 256 and base % 256 == 0
    cm = rkv.make_config(redundancy_mode=rkv.RKV_RED_MAX)
    assert rkv.rkv_workspace_size(cm, 32, 1, 1152) >= base + 32 * 8 * 1152 * 4
    assert rkv.rkv_workspace_size(rkv.make_config(head_dim=64), 1, 1, 100) == 0
    assert rkv.rkv_workspace_size(c, 0, 1, 100) == 0


# Fake device addresses: validation rejects these calls before any CUDA call.
A = 1 << 40


def _step(cfg, n_layers=2, batch=1, cap=1152, k=None, v=None, q=None, cur=A + 7 * 4096,
          ws=A + 9 * 4096, ws_bytes=1 << 20, budgets=None):
    L = rkv._lib
    arr = ctypes.c_void_p * n_layers
    k = arr(*(k or [A + i * (1 << 30) for i in range(n_layers)]))
    v = arr(*(v or [A + (1 << 36) + i * (1 << 30) for i in range(n_layers)]))
    q = arr(*(q or [A + (1 << 37) + i * (1 << 20) for i in range(n_layers)]))
    return L.rkv_compress_step(ctypes.byref(cfg), n_layers, batch, cap, k, v, q, budgets, None,
                               cur, None, ws, ws_bytes, None)


def test_compress_step_host_validation():
    c = rkv.make_config()
    assert rkv._lib.rkv_compress_step(None, 1, 1, 1152, None, None, None, None, None, None, None,
                                      None, 0, None) == -1
    assert _step(rkv.make_config(budget=0)) == rkv.RKV_STATUS_DISABLED
    assert _step(rkv.make_config(buffer=0)) == rkv.RKV_STATUS_DISABLED
    assert _step(rkv.make_config(head_dim=64)) == -6
    assert _step(rkv.make_config(n_q_heads=30)) == -2
    assert _step(rkv.make_config(window=0)) == -2
    assert _step(rkv.make_config(n_q_heads=8 * 16, window=8)) == -6      # G*w = 128 > 64
    assert _step(rkv.make_config(mix_lambda=float("nan"))) == -2
    assert _step(c, ws=None) == -5
    assert _step(c, cur=None) == -1
    assert _step(rkv.make_config(budget=1200), cap=1152) == -2           # budget >= cap
    assert _step(rkv.make_config(budget=4, window=8)) == -2              # budget < window
    assert _step(c, k=[A + 8, A + (1 << 30)]) == -3                      # misaligned K
    assert _step(c, k=[A, A + (1 << 30)], v=[A + 4096, A + (1 << 31)]) == -4   # K overlaps V
    assert _step(c, ws_bytes=16) == -5
    assert _step(c, ws=A + 9 * 4096 + 16) == -3                          # workspace 256-aligned


def test_per_head_entry_points_host_validation():
    L = rkv._lib
    c = rkv.make_config()
    cfgp = ctypes.byref(c)
    # importance: null output, bad stride, n_tokens <= window, small workspace
    assert L.rkv_score_importance(cfgp, A, A + 4096, 1152 * 128, 1152, None, None, A, 4096, None) == -1
    assert L.rkv_score_importance(cfgp, A, A + 4096, 1152 * 128 + 3, 1152, A, None, A, 4096, None) == -3
    assert L.rkv_score_importance(cfgp, A, A + 4096, 1152 * 128, 8, A, None, A, 4096, None) == -2
    assert L.rkv_score_importance(cfgp, A, A + 4096, 1152 * 128, 1152, A, None, A, 8, None) == -5
    # redundancy: nothing to write
    assert L.rkv_score_redundancy(cfgp, A, 1152 * 128, 1152, None, None, A, 4096, None) == -1
    # select: budget above n_tokens; disabled budget
    assert L.rkv_select_topk(cfgp, A, A, 1000, A, None, A, 4096, None) == -2
    assert L.rkv_select_topk(ctypes.byref(rkv.make_config(budget=0)), A, A, 1000, A, None, A,
                             4096, None) == 1
    # compaction: one of K/V in place only, overlapping out-of-place buffers, bad alignment
    hs = 1152 * 128
    assert L.rkv_compact_kv(cfgp, A, A + (1 << 32), A + (1 << 34), A, A + (1 << 33), hs, 1152,
                            A + (1 << 35), 4096, None) == -4
    assert L.rkv_compact_kv(cfgp, A, A + (1 << 32), A + (1 << 34), A + 4096, A + (1 << 33), hs,
                            1152, A + (1 << 35), 4096, None) == -4
    assert L.rkv_compact_kv(cfgp, A + 2, A + (1 << 32), A + (1 << 34), A + 2, A + (1 << 32), hs,
                            1152, A + (1 << 35), 4096, None) == -3


def test_step_shape_query():
    """Few units: a cluster per unit, two CTAs per SM.  One unit per SM or more:
    one CTA per unit, two CTAs per SM at the 8B-model shapes."""
    cfg = rkv.make_config()
    cs, rows, smem = rkv.rkv_query_step_shape(cfg, 8, 1152)
    assert (cs, rows) == (8, 144) and smem <= 233472 // 2 - 1024
    cs, rows, smem = rkv.rkv_query_step_shape(cfg, 256, 1152)
    assert (cs, rows) == (1, 1152) and smem <= 233472 // 2 - 1024
    cs, rows, smem = rkv.rkv_query_step_shape(rkv.make_config(2048, n_q_heads=40), 8, 2176)
    assert rows * cs >= 2176 and smem <= 233472 // 2 - 1024
    cs, rows, smem = rkv.rkv_query_step_shape(rkv.make_config(2048, n_q_heads=40), 6144, 2176)
    assert (cs, rows) == (1, 2176) and smem <= 232448
    # a unit too long for either kernel's shared memory
    with pytest.raises(rkv.RkvError):
        rkv.rkv_query_step_shape(cfg, 6144, 8000)
    with pytest.raises(rkv.RkvError):
        rkv.rkv_query_step_shape(rkv.make_config(head_dim=64), 8, 1152)
    with pytest.raises(rkv.RkvError):
        rkv.rkv_query_step_shape(cfg, 0, 1152)


def test_shared_selection_host_validation():
    L = rkv._lib
    c = rkv.make_config()
    cfgp = ctypes.byref(c)
    arr = ctypes.c_void_p * 2
    k = arr(A, A + (1 << 30))
    v = arr(A + (1 << 36), A + (1 << 36) + (1 << 30))
    q = arr(A + (1 << 37), A + (1 << 37) + (1 << 20))
    need = rkv.rkv_workspace_size_shared(c, 2, 1, 1152)
    assert need > rkv.rkv_workspace_size(c, 2, 1, 1152)
    ws, cur, z = A + (1 << 38), A + 7 * 4096, A + (1 << 39)
    # score: missing q, z or workspace; workspace too small; misaligned z
    assert L.rkv_score_shared(cfgp, 2, 1, 1152, k, None, None, None, cur, z, ws, need, None) == -1
    assert L.rkv_score_shared(cfgp, 2, 1, 1152, k, q, None, None, cur, None, ws, need, None) == -1
    assert L.rkv_score_shared(cfgp, 2, 1, 1152, k, q, None, None, cur, z, None, need, None) == -5
    # (the size includes 256 bytes of room for the order of the sequences, which a call
    # can do without; 512 short is below what it needs)
    assert L.rkv_score_shared(cfgp, 2, 1, 1152, k, q, None, None, cur, z, ws, need - 512, None) == -5
    assert L.rkv_score_shared(cfgp, 2, 1, 1152, k, q, None, None, cur, z + 4, ws, need, None) == -3
    assert L.rkv_score_shared(ctypes.byref(rkv.make_config(buffer=0)), 2, 1, 1152, k, q, None,
                              None, cur, z, ws, need, None) == 1
    # select + compact: K overlapping V, caches too long for one CTA per head
    vbad = arr(A + 4096, A + (1 << 36))
    assert L.rkv_select_compact_shared(cfgp, 2, 1, 1152, k, vbad, None, cur, z, None, ws, need,
                                       None) == -4
    big = rkv.rkv_workspace_size_shared(c, 2, 1, 9000)
    assert L.rkv_select_compact_shared(cfgp, 2, 1, 9000, k, v, None, cur, z, None, ws, big,
                                       None) == -6


def test_ragged_step_host_validation():
    L = rkv._lib
    c = rkv.make_config()
    cfgp = ctypes.byref(c)
    arr = ctypes.c_void_p * 2
    k = arr(A, A + (1 << 34))
    v = arr(A + (1 << 36), A + (1 << 36) + (1 << 34))
    q = arr(A + (1 << 37), A + (1 << 37) + (1 << 20))
    cur, ws = A + 7 * 4096, A + (1 << 38)
    need = rkv.rkv_workspace_size(c, 2, 4, 2176)

    def call(rg=None, cfg=cfgp, kk=k, vv=v, ws_=ws, ws_bytes=need, opts=None):
        if rg is None:
            rg = rkv.rkv_ragged_kv(A + (1 << 39), A + (1 << 39) + 4096, 4 * 8 * 2176, 2176)
        return L.rkv_compress_step_ragged(cfg, 2, 4, ctypes.byref(rg), kk, vv, q, None, None,
                                          cur, opts, ws_, ws_bytes, None)

    assert L.rkv_compress_step_ragged(cfgp, 2, 4, None, k, v, q, None, None, cur, None, ws,
                                      need, None) == -1
    assert call(rkv.rkv_ragged_kv(None, A, 100, 2176)) == -1                 # no seq_row
    assert call(rkv.rkv_ragged_kv(A + 4, A, 100000, 2176)) == -3             # seq_row not 8-aligned
    assert call(rkv.rkv_ragged_kv(A, A, 1 << 31, 2176)) == -6                # rows past int32
    assert call(rkv.rkv_ragged_kv(A, A, 100000, 1)) == -2                    # max_cap < 2
    assert call(rkv.rkv_ragged_kv(A, A, 100000, 1000)) == -2                 # budget >= max_cap
    assert call(rkv.rkv_ragged_kv(A, A, 100000, 9000)) == -6                 # one CTA cannot hold it
    assert call(cfg=ctypes.byref(rkv.make_config(buffer=0))) == 1            # disabled
    assert call(ws_=None) == -5
    assert call(ws_bytes=need - 512) == -5                                   # below the required part
    assert call(ws_=ws + 16) == -3
    assert call(vv=arr(A + 4096, A + (1 << 36))) == -4                       # K pool overlaps V pool
    opts = rkv.rkv_step_options(None, None, None, None, 8)
    assert call(opts=ctypes.byref(opts)) == -6                               # clusters unsupported


def test_ragged_layout_helpers():
    import torch
    from rkv_synth import pack_ragged, unpack_ragged
    rows, total = rkv.ragged_rows([10, 3, 7], 2)
    assert rows == [0, 20, 26] and total == 40
    X = torch.arange(2 * 3 * 2 * 10 * 4, dtype=torch.float32).reshape(2, 3, 2, 10, 4)
    P = pack_ragged(X, [10, 3, 7])
    assert P.shape == (2, 40, 4)
    assert torch.equal(P[:, 20:23], X[:, 1, 0, :3]) and torch.equal(P[:, 23:26], X[:, 1, 1, :3])
    Y = unpack_ragged(P, [10, 3, 7], 2, 10)
    assert torch.equal(Y[:, 0], X[:, 0])
    assert torch.equal(Y[:, 2, :, :7], X[:, 2, :, :7]) and not Y[:, 2, :, 7:].any()


def test_max_redundancy_row_limit():
    """MAX redundancy keeps per-row keys and norms of a whole unit in the similarity
    kernel's shared memory: caches longer than 7680 rows are refused on the host."""
    cm = rkv.make_config(redundancy_mode=rkv.RKV_RED_MAX)
    assert _step(cm, cap=7808, ws_bytes=1 << 30) == -6
