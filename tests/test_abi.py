"""The C-ABI library loads, exports every symbol include/gqe.h declares, and
rejects bad arguments on the host before launching anything (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "gqe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gq[ae]_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def rsq():
    from routed_sparse_query_b200 import build
    build.build()
    import routed_sparse_query_b200 as m
    return m


def test_header_declares_the_entry_points():
    fns = _header_functions()
    for name in ("gqe_router_topk", "gqe_dispatch", "gqe_attention_fwd", "gqe_output_proj",
                 "gqa_dense_fwd", "gqe_kv_proj", "gqe_layer_fwd", "gqe_workspace_bytes"):
        assert name in fns


def test_library_exports_every_declared_symbol(rsq):
    lib = ctypes.CDLL(rsq.LIB_PATH)
    missing = [f for f in _header_functions() if not hasattr(lib, f)]
    assert not missing, missing
    assert set(rsq.EXPORTED) == set(_header_functions())


def test_version_and_status_strings(rsq):
    assert rsq.gqe_version() >= 100
    assert rsq.gqe_status_string(0) == "ok"
    assert "timed out" in rsq.gqe_status_string(rsq.GQE_ERR_TIMEOUT)


def _cfg(rsq, **kw):
    base = dict(B=1, T=2048, d_model=1024, G=8, M=2, k=1, d_head=64)
    base.update(kw)
    return rsq.GQEConfig(base["B"], base["T"], base["d_model"], base["G"], base["M"], base["k"],
                         base["d_head"], 0)


@pytest.mark.parametrize("bad", [dict(k=3), dict(k=0), dict(T=0), dict(B=0), dict(d_model=1000),
                                 dict(G=0)])
def test_invalid_configs_have_no_workspace(rsq, bad):
    assert rsq.gqe_workspace_bytes(_cfg(rsq, **bad), rsq.GQE_WS_LAYER) == 0


def test_unsupported_head_dim(rsq):
    lib = rsq.lib()
    c = _cfg(rsq, d_head=128)
    st = lib.gqe_router_topk(ctypes.byref(c), None, None, None, None, None, None, None)
    assert st == rsq.GQE_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected_on_host(rsq):
    lib = rsq.lib()
    c = _cfg(rsq)
    assert lib.gqe_router_topk(ctypes.byref(c), None, None, None, None, None, None,
                               None) == rsq.GQE_ERR_INVALID
    p = ctypes.c_void_p(0x1000_0008)  # not 16-byte aligned; never dereferenced
    assert lib.gqe_kv_proj(ctypes.byref(c), p, p, p, p, p, None) == rsq.GQE_ERR_INVALID
    assert lib.gqe_selftest_wait_timeout(10, None) == rsq.GQE_ERR_INVALID


def test_workspace_too_small_rejected_on_host(rsq):
    lib = rsq.lib()
    c = _cfg(rsq)
    need = rsq.gqe_workspace_bytes(c, rsq.GQE_WS_LAYER)
    assert need > 0
    p = ctypes.c_void_p(0x1000_0000)  # aligned; never dereferenced
    st = lib.gqe_layer_fwd(ctypes.byref(c), p, p, None, p, p, p, p, p, p, p, need - 1, None)
    assert st == rsq.GQE_ERR_WORKSPACE


def test_workspace_sizes_cover_items(rsq):
    c = _cfg(rsq)
    R, G, k, dh = 2048, 8, 1, 64
    total = rsq.gqe_workspace_bytes(c, rsq.GQE_WS_LAYER)
    slots = rsq.gqe_workspace_offset(c, rsq.GQE_WS_LAYER, "slots")
    assert slots + R * (k * G + 2) * dh * 2 <= total
    assert rsq.gqe_workspace_offset(c, rsq.GQE_WS_LAYER, "K") % 256 == 0
    assert rsq.gqe_workspace_bytes(c, rsq.GQE_WS_DENSE) >= R * 16 * dh * 2 * 2


def test_router_staging_limit(rsq):
    # The router stages W_r (fp32, zero-padded to a power-of-two column count)
    # in shared memory: 32 experts at d_model = 1024 (the expert-pool
    # workloads) fit, 64 experts at d_model = 1024 (256 KB of W_r) do not and
    # are refused on the host, 64 experts at d_model = 256 fit again.
    ws = rsq.GQE_WS_LAYER
    assert rsq.gqe_workspace_bytes(_cfg(rsq, G=8, M=4, k=2), ws) > 0
    assert rsq.gqe_workspace_bytes(_cfg(rsq, G=8, M=8), ws) == 0
    assert rsq.gqe_workspace_bytes(_cfg(rsq, G=8, M=8, d_model=256), ws) > 0
    lib = rsq.lib()
    c = _cfg(rsq, G=8, M=8)
    assert lib.gqe_router_topk(ctypes.byref(c), None, None, None, None, None, None,
                               None) == rsq.GQE_ERR_UNSUPPORTED


def test_attention_split_kv_plan(rsq):
    # Split-KV (and its workspace of partial rows) only when the query-tile
    # pairs of all streams are fewer than the SMs: 9 streams x 8 pairs at
    # T = 2048 are split, 9 x 128 pairs at T = 32768 are not (the workspace is
    # then the 256-byte minimum).
    ws = rsq.GQE_WS_ATTENTION
    small = rsq.gqe_workspace_bytes(_cfg(rsq, T=2048), ws)
    large = rsq.gqe_workspace_bytes(_cfg(rsq, T=32768), ws)
    assert large == 256
    rows = 9 * 16 * 2 * 128  # streams x items (chunk of 5 KV tiles: 16 per stream) x 2 tiles x 128 rows
    assert small >= rows * 64 * 4 + rows * 8  # fp32 partial O rows and (m, l) pairs


def test_output_construction_flags(rsq):
    # At most one output construction; the ablation ones (no weighted slot, no
    # shared head) have kG slots, the others kG+2; the decode step takes the
    # layer's construction only.
    c = _cfg(rsq)
    R, G, k, dh = 2048, 8, 1, 64
    for flags, S in ((0, k * G + 2), (rsq.GQE_FLAG_SLOT_GROUP_MEAN, k * G + 2),
                     (rsq.GQE_FLAG_OUT_HARD, k * G), (rsq.GQE_FLAG_OUT_WEIGHTED_CONCAT, k * G)):
        c.flags = flags
        total = rsq.gqe_workspace_bytes(c, rsq.GQE_WS_LAYER)
        slots = rsq.gqe_workspace_offset(c, rsq.GQE_WS_LAYER, "slots")
        assert total > 0 and slots + R * S * dh * 2 <= total
        assert rsq.gqe_workspace_bytes(c, rsq.GQE_WS_DECODE) == (0 if flags else
                                                                 rsq.gqe_workspace_bytes(c, rsq.GQE_WS_DECODE))
    c.flags = rsq.GQE_FLAG_OUT_HARD | rsq.GQE_FLAG_SLOT_GROUP_MEAN
    assert rsq.gqe_workspace_bytes(c, rsq.GQE_WS_LAYER) == 0
    lib = rsq.lib()
    assert lib.gqe_router_topk(ctypes.byref(c), None, None, None, None, None, None,
                               None) == rsq.GQE_ERR_INVALID
    c.flags = 1 << 7  # unknown bit
    assert rsq.gqe_workspace_bytes(c, rsq.GQE_WS_LAYER) == 0
    # The ablation constructions take no shared head: Qs / W_qs may be NULL.
    c.flags = rsq.GQE_FLAG_OUT_HARD
    p = ctypes.c_void_p(0x1000_0000)  # aligned; never dereferenced (workspace too small)
    st = lib.gqe_dispatch(ctypes.byref(c), p, p, p, None, p, p, p, p, p, None, p, 16, None)
    assert st == rsq.GQE_ERR_WORKSPACE
