"""The C ABI library on the host: it loads, exports every function
include/basiskv.h declares, and its host-side validation rejects bad arguments
before launching anything.

The calls below pass made-up device addresses, which only the entry points'
own checks keep from reaching a kernel.  So these tests always run in a
process that sees no GPU: in place when none is visible, otherwise in a child
process started with CUDA_VISIBLE_DEVICES empty, where a check that let a call
through would fail with a CUDA error instead of touching device memory."""
import ctypes
import os
import re
import subprocess
import sys

import pytest
import torch

from long_context_decode_basiskv_b200 import binding as bk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GPU_VISIBLE = os.environ.get("CUDA_VISIBLE_DEVICES") != "" and torch.cuda.is_available()


def test_host_checks_in_a_process_without_gpu():
    """With a GPU visible, run this file again in a child process that sees none."""
    if not GPU_VISIBLE:
        pytest.skip("no GPU visible: the checks run in this process")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "not gpu",
                        os.path.abspath(__file__)], env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def _declared():
    src = open(os.path.join(ROOT, "include", "basiskv.h")).read()
    return sorted(set(re.findall(r"BASISKV_API\s+[\w\s\*]+?\b(basiskv_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    if GPU_VISIBLE:
        pytest.skip("a GPU is visible: these calls run in test_host_checks_in_a_process_without_gpu")
    if not os.path.exists(bk.LIB_PATH):
        from long_context_decode_basiskv_b200 import build
        build.build()
    return bk.lib()


def test_header_declarations_match_binding():
    # reads files only
    assert _declared() == sorted(bk.SYMBOLS)


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_version_and_status_strings(L):
    assert L.basiskv_abi_version() == 4
    assert L.basiskv_status_string(0) == b"ok"
    assert L.basiskv_status_string(4).startswith(b"workspace")
    assert L.basiskv_status_string(99) == b"unknown status"


def _cfg(**kw):
    base = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, rank_v=64, rank_k=32, page_size=16,
                hidden=4096, top_k=128, dtype=bk.BF16)
    base.update(kw)
    return bk.CConfig(*[base[f] for f, _ in bk.CConfig._fields_])


def test_workspace_bytes(L):
    n = L.basiskv_workspace_bytes(ctypes.byref(_cfg()), 8, 2048)
    assert n >= 8 * 32 * 2048 * 4          # at least the routing scores
    assert L.basiskv_workspace_bytes(ctypes.byref(_cfg(head_dim=96)), 8, 2048) == 0
    assert L.basiskv_workspace_bytes(None, 8, 2048) == 0


@pytest.mark.parametrize("bad,status", [
    (dict(num_q_heads=30), bk.ERR_INVALID_ARG),        # Hq % Hkv != 0
    (dict(head_dim=96), bk.ERR_UNSUPPORTED),
    (dict(page_size=8), bk.ERR_UNSUPPORTED),
    (dict(rank_v=0), bk.ERR_INVALID_ARG),
    (dict(top_k=1023), bk.ERR_UNSUPPORTED),
    (dict(num_q_heads=48, num_kv_heads=3), bk.ERR_UNSUPPORTED),   # G = 16
    (dict(dtype=7), bk.ERR_INVALID_ARG),
])
def test_config_validation(L, bad, status):
    cfg = _cfg(**bad)
    cache = bk.CCache(16, 16, 16, 16, 16, 16, 10, 10)   # never dereferenced: validation fails first
    st = L.basiskv_route(ctypes.byref(cfg), ctypes.byref(cache), 16, 1, 16, 16, None, 16, 1 << 30, 16, None)
    assert st == status


def test_null_and_misaligned_pointers(L):
    cfg = _cfg()
    good = bk.CCache(256, 256, 256, 256, 256, 256, 10, 10)
    assert L.basiskv_route(ctypes.byref(cfg), None, 256, 1, 256, 256, None, 256, 1 << 30, 256, None) == bk.ERR_INVALID_ARG
    misaligned = bk.CCache(264, 256, 256, 256, 256, 256, 10, 10)
    assert L.basiskv_route(ctypes.byref(cfg), ctypes.byref(misaligned), 256, 1, 256, 256, None, 256,
                           1 << 30, 256, None) == bk.ERR_INVALID_ARG
    # workspace too small
    assert L.basiskv_route(ctypes.byref(cfg), ctypes.byref(good), 256, 1, 256, 256, None, 256, 16, 256,
                           None) == bk.ERR_WORKSPACE
    assert L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(good), 256, 1, 256, 256, 256, None, 0,
                                 256, None) == bk.ERR_WORKSPACE
    # err flag required
    f = bk.CFactors(256, 256, 256, 256)
    assert L.basiskv_append(ctypes.byref(cfg), ctypes.byref(good), ctypes.byref(f), 256, 256, 1, 1, None,
                            None) == bk.ERR_INVALID_ARG
    # too many pages for the routing kernel
    big = bk.CCache(256, 256, 256, 256, 256, 256, 10, 1 << 20)
    assert L.basiskv_route(ctypes.byref(cfg), ctypes.byref(big), 256, 1, 256, 256, None, 256, 1 << 40, 256,
                           None) == bk.ERR_UNSUPPORTED


def test_empty_batch_is_a_no_op(L):
    cfg = _cfg()
    good = bk.CCache(256, 256, 256, 256, 256, 256, 10, 10)
    f = bk.CFactors(256, 256, 256, 256)
    assert L.basiskv_append(ctypes.byref(cfg), ctypes.byref(good), ctypes.byref(f), 256, 256, 0, 1, 256,
                            None) == bk.OK
    assert L.basiskv_route(ctypes.byref(cfg), ctypes.byref(good), 256, 0, 256, 256, None, None, 0, 256,
                           None) == bk.OK
    assert L.basiskv_out_proj(ctypes.byref(cfg), ctypes.byref(f), 256, 0, 256, None, 0, None) == bk.OK


@pytest.mark.parametrize("bad,status", [
    (dict(rank_k=80), bk.ERR_UNSUPPORTED),             # residual rank above 64
    (dict(rank_v=160, head_dim=128), bk.ERR_INVALID_ARG),  # latent rank above d
    (dict(hidden=4100), bk.ERR_UNSUPPORTED),           # hidden not a multiple of 16
    (dict(top_k=0), bk.ERR_INVALID_ARG),
    (dict(num_kv_heads=0), bk.ERR_INVALID_ARG),
])
def test_more_config_limits(L, bad, status):
    cfg = _cfg(**bad)
    cache = bk.CCache(16, 16, 16, 16, 16, 16, 10, 10)
    st = L.basiskv_route(ctypes.byref(cfg), ctypes.byref(cache), 16, 1, 16, 16, None, 16, 1 << 30, 16, None)
    assert st == status


def test_append_longer_than_the_block_table(L):
    cfg = _cfg()
    cache = bk.CCache(256, 256, 256, 256, 256, 256, 10, 4)      # 4 pages of 16 tokens
    f = bk.CFactors(256, 256, 256, 256)
    assert L.basiskv_append(ctypes.byref(cfg), ctypes.byref(cache), ctypes.byref(f), 256, 256, 1, 65, 256,
                            None) == bk.ERR_INVALID_ARG
    misaligned = bk.CFactors(264, 256, 256, 256)
    assert L.basiskv_append(ctypes.byref(cfg), ctypes.byref(cache), ctypes.byref(misaligned), 256, 256, 1, 1,
                            256, None) == bk.ERR_INVALID_ARG


def test_out_proj_pointer_checks(L):
    cfg = _cfg()
    f = bk.CFactors(256, 256, 256, 256)
    assert L.basiskv_out_proj(ctypes.byref(cfg), None, 256, 1, 256, None, 0, None) == bk.ERR_INVALID_ARG
    assert L.basiskv_out_proj(ctypes.byref(cfg), ctypes.byref(bk.CFactors(256, 256, 256, 0)), 256, 1, 256, None,
                              0, None) == bk.ERR_INVALID_ARG           # no fused factor
    assert L.basiskv_out_proj(ctypes.byref(cfg), ctypes.byref(f), 260, 1, 256, None, 0, None) == bk.ERR_INVALID_ARG
    assert L.basiskv_out_proj(ctypes.byref(cfg), ctypes.byref(f), 256, 1, None, None, 0, None) == bk.ERR_INVALID_ARG


def test_workspace_grows_with_the_problem(L):
    cfg = ctypes.byref(_cfg())
    a = L.basiskv_workspace_bytes(cfg, 8, 2048)
    assert L.basiskv_workspace_bytes(cfg, 16, 2048) > a
    assert L.basiskv_workspace_bytes(cfg, 8, 4096) > a
    assert L.basiskv_workspace_bytes(ctypes.byref(_cfg(dtype=bk.F32)), 8, 2048) > 0
    assert L.basiskv_workspace_bytes(cfg, 8, 0) == 0
    assert L.basiskv_workspace_bytes(cfg, -1, 2048) == 0


def test_noalloc_refuses_shapes_beyond_its_scratch(L):
    # 1024 sequences x 64 query heads need far more split scratch than the fixed 16 MiB
    cfg = _cfg(num_q_heads=64, num_kv_heads=8, rank_v=128, top_k=256)
    cache = bk.CCache(256, 256, 256, 256, 256, 256, 10, 4096)
    st = L.basiskv_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(cache), 256, 1024, 256, 256, 256, 256, None)
    assert st == bk.ERR_WORKSPACE


def test_route_group_checks(L):
    """basiskv_route_group: only GROUP_SUM / GROUP_MAX are reductions; the rest of its
    validation is basiskv_route's (an empty batch launches nothing)."""
    cfg = _cfg()
    good = bk.CCache(256, 256, 256, 256, 256, 256, 10, 10)
    for bad in (0, 3, -1):
        assert L.basiskv_route_group(ctypes.byref(cfg), ctypes.byref(good), 256, 1, bad, 256, 256, None, 256,
                                     1 << 30, 256, None) == bk.ERR_INVALID_ARG
    for red in (bk.GROUP_SUM, bk.GROUP_MAX):
        assert L.basiskv_route_group(ctypes.byref(cfg), ctypes.byref(good), 256, 0, red, 256, 256, None, None,
                                     0, 256, None) == bk.OK
        assert L.basiskv_route_group(ctypes.byref(cfg), None, 256, 1, red, 256, 256, None, 256, 1 << 30, 256,
                                     None) == bk.ERR_INVALID_ARG
        assert L.basiskv_route_group(ctypes.byref(cfg), ctypes.byref(good), 260, 1, red, 256, 256, None, 256,
                                     1 << 30, 256, None) == bk.ERR_INVALID_ARG   # misaligned q


def test_append_route_checks(L):
    """basiskv_append_route: the append's and the route's checks, all before any launch
    (reduce 0 = per head, else GROUP_SUM / GROUP_MAX)."""
    cfg = _cfg()
    good = bk.CCache(256, 256, 256, 256, 256, 256, 10, 10)
    f = bk.CFactors(256, 256, 256, 256)

    def call(cache=good, fac=f, k=256, v=256, q=256, batch=1, reduce=0, sel=256, ws=256, ws_bytes=1 << 30, err=256):
        return L.basiskv_append_route(ctypes.byref(cfg), ctypes.byref(cache) if cache else None,
                                      ctypes.byref(fac) if fac else None, k, v, q, batch, reduce, sel, 256, ws,
                                      ws_bytes, err, None)

    for bad in (3, -1, 7):
        assert call(reduce=bad) == bk.ERR_INVALID_ARG
    assert call(batch=0) == bk.OK                                  # nothing to do
    assert call(cache=None) == bk.ERR_INVALID_ARG
    assert call(fac=None) == bk.ERR_INVALID_ARG
    assert call(k=None) == bk.ERR_INVALID_ARG
    assert call(err=None) == bk.ERR_INVALID_ARG
    assert call(q=260) == bk.ERR_INVALID_ARG                       # misaligned q
    assert call(ws=None) == bk.ERR_WORKSPACE
    assert call(ws_bytes=64) == bk.ERR_WORKSPACE
    assert call(fac=bk.CFactors(260, 256, 256, 256)) == bk.ERR_INVALID_ARG   # misaligned A


def test_prefill_checks(L):
    """basiskv_prefill: bf16 with ranks that are multiples of 16 only; otherwise basiskv_append's checks."""
    good = bk.CCache(256, 256, 256, 256, 256, 256, 10, 10)
    f = bk.CFactors(256, 256, 256, 256)
    for bad in (dict(dtype=bk.F32), dict(rank_k=8), dict(rank_v=24), dict(head_dim=96, rank_v=32),
                dict(head_dim=64, rank_v=32)):
        cfg = _cfg(**bad)
        assert L.basiskv_prefill(ctypes.byref(cfg), ctypes.byref(good), ctypes.byref(f), 256, 256, 1, 64, 256,
                                 None) == bk.ERR_UNSUPPORTED, bad
    cfg = _cfg()
    assert L.basiskv_prefill(ctypes.byref(cfg), ctypes.byref(good), ctypes.byref(f), 256, 256, 0, 64, 256,
                             None) == bk.OK
    assert L.basiskv_prefill(ctypes.byref(cfg), ctypes.byref(good), ctypes.byref(f), 264, 256, 1, 64, 256,
                             None) == bk.ERR_INVALID_ARG                       # misaligned k_new
    assert L.basiskv_prefill(ctypes.byref(cfg), ctypes.byref(good), ctypes.byref(f), 256, 256, 1, 64, None,
                             None) == bk.ERR_INVALID_ARG                       # no error flag
    assert L.basiskv_prefill(ctypes.byref(cfg), ctypes.byref(good), ctypes.byref(f), 256, 256, 1, 161, 256,
                             None) == bk.ERR_INVALID_ARG                       # more tokens than the block table holds


@pytest.mark.parametrize("bad,status", [
    (dict(dtype=7), bk.ERR_INVALID_ARG),
    (dict(head_dim=96), bk.ERR_UNSUPPORTED),
    (dict(num_q_heads=30), bk.ERR_INVALID_ARG),
])
def test_noalloc_validates_like_decode_attn(L, bad, status):
    """The allocation-free call refuses a bad configuration exactly as the workspace call does,
    before it looks at the size of its scratch."""
    cfg = _cfg(**bad)
    cache = bk.CCache(256, 256, 256, 256, 256, 256, 10, 10)
    a = L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(cache), 256, 1, 256, 256, 256, 256, 1 << 30, 256, None)
    b = L.basiskv_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(cache), 256, 1, 256, 256, 256, 256, None)
    assert a == b == status


def test_noalloc_and_decode_attn_share_cache_limits(L):
    cfg = _cfg()
    big = bk.CCache(256, 256, 256, 256, 256, 256, 10, 49153)          # more pages than routing supports
    assert L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(big), 256, 1, 256, 256, 256, 256, 1 << 40, 256,
                                 None) == bk.ERR_UNSUPPORTED
    assert L.basiskv_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(big), 256, 1, 256, 256, 256, 256,
                                         None) == bk.ERR_UNSUPPORTED
    many = bk.CCache(256, 256, 256, 256, 256, 256, 1 << 24, 10)       # page ids beyond 24 bits
    assert L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(many), 256, 1, 256, 256, 256, 256, 1 << 40, 256,
                                 None) == bk.ERR_UNSUPPORTED
    assert L.basiskv_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(many), 256, 1, 256, 256, 256, 256,
                                         None) == bk.ERR_UNSUPPORTED
    # no summary pointer: attention does not read summaries, so both calls accept it up to the workspace
    nosum = bk.CCache(256, 256, 256, 0, 256, 256, 10, 10)
    assert L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(nosum), 256, 1, 256, 256, 256, None, 0, 256,
                                 None) == bk.ERR_WORKSPACE


def test_selection_pointers_come_in_pairs(L):
    cfg = _cfg()
    good = bk.CCache(256, 256, 256, 256, 256, 256, 10, 10)
    # sel without sel_cnt (or the reverse) is refused by both calls
    assert L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(good), 256, 1, 256, None, 256, 256, 1 << 30, 256,
                                 None) == bk.ERR_INVALID_ARG
    assert L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(good), 256, 1, None, 256, 256, 256, 1 << 30, 256,
                                 None) == bk.ERR_INVALID_ARG
    assert L.basiskv_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(good), 256, 1, 256, None, 256, 256,
                                         None) == bk.ERR_INVALID_ARG
    # the allocation-free call has no routing workspace to take a selection from
    assert L.basiskv_decode_attn_noalloc(ctypes.byref(cfg), ctypes.byref(good), 256, 1, None, None, 256, 256,
                                         None) == bk.ERR_INVALID_ARG
    # with both NULL the workspace call attends over the routing call's lists: workspace still required
    assert L.basiskv_decode_attn(ctypes.byref(cfg), ctypes.byref(good), 256, 1, None, None, 256, None, 0, 256,
                                 None) == bk.ERR_WORKSPACE
