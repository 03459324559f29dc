"""The C ABI without a GPU: the library loads, exports every symbol that
include/tb.h declares, sizes workspaces, and rejects bad arguments on the host
before any CUDA call."""
import ctypes
import os
import re

import pytest
import torch  # noqa: F401  (loads the CUDA runtime libtb links against)

from query_aware_sparse_tb_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "tb.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tb_[a-z_0-9]+)\s*\(", src)))


def test_exports_match_header(lib):
    declared = _declared()
    assert declared, "no declarations found"
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in tb.h but not exported"
    assert sorted(_lib.EXPORTS) == declared


def _header_constants():
    src = open(os.path.join(ROOT, "include", "tb.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    consts = {m.group(1): int(m.group(2), 0)
              for m in re.finditer(r"^#define (TB_[A-Z_]+)\s+(0x[0-9a-fA-F]+|\d+)u?\s*$", src, flags=re.M)}
    consts.update({m.group(1): int(m.group(2)) for m in re.finditer(r"\b(TB_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", src)})
    return consts


def test_binding_constants_match_header(lib):
    h = _header_constants()
    for name in ("TB_OK", "TB_ERR_INVALID_ARG", "TB_ERR_UNSUPPORTED", "TB_ERR_CUDA", "TB_ERR_WORKSPACE",
                 "TB_ERR_DEVICE_FLAG", "TB_FLAG_CTX_RANGE", "TB_FLAG_TIMEOUT", "TB_FLAG_IDX_OVERFLOW",
                 "TB_FLAG_BAD_CACHE", "TB_ATTN_WAIT_ALL", "TB_ATTN_PREFETCH_KV"):
        assert getattr(_lib, name) == h[name], name
        if name.startswith(("TB_OK", "TB_ERR_")):
            assert lib.tb_status_str(h[name]) == name.encode()
    assert _lib.TB_GROUP_REDUCE == {"max": h["TB_GROUP_MAX"], "sum": h["TB_GROUP_SUM"]}
    assert lib.tb_abi_version() == h["TB_ABI_VERSION"] == _lib.TB_ABI_VERSION


def test_version_and_strings(lib):
    assert lib.tb_abi_version() == 10
    assert lib.tb_status_str(0) == b"TB_OK"
    assert lib.tb_status_str(2) == b"TB_ERR_UNSUPPORTED"


def _d(**kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, d_proj=32, ctx_cap=65792)
    base.update(kw)
    return _lib.TbDims(*[base[k] for k in ("batch", "n_q_heads", "n_kv_heads", "head_dim", "d_proj", "ctx_cap")])


def test_workspace_sizes(lib):
    d = _d()
    a = lib.tb_attn_workspace_bytes(ctypes.byref(d))
    s = lib.tb_score_select_workspace_bytes(ctypes.byref(d))
    assert a > 256 and s > 256
    # selection workspace holds at least keys (4 B) + candidates (8 B) per (head, position)
    assert s >= 32 * 65792 * 12
    assert lib.tb_attn_workspace_bytes(ctypes.byref(_d(head_dim=96))) == 0
    assert lib.tb_score_select_workspace_bytes(ctypes.byref(_d(d_proj=24))) == 0
    assert lib.tb_score_select_workspace_bytes(ctypes.byref(_d(ctx_cap=(1 << 19) + 1))) == 0
    assert lib.tb_predict_queries_workspace_bytes(1, 4096, 1024, 4096) > 0
    assert lib.tb_predict_queries_workspace_bytes(17, 4096, 1024, 4096) == 0
    assert lib.tb_project_keys_workspace_bytes() == 256


FAKE = 1 << 20          # 16-byte aligned, never dereferenced: validation fails first
MIS = FAKE + 8          # misaligned


def test_attention_rejects_bad_arguments(lib):
    d = _d()
    ws_bytes = lib.tb_attn_workspace_bytes(ctypes.byref(d))
    ok_args = dict(Q=FAKE, K=FAKE, V=FAKE, ctx=FAKE, out=FAKE, ws=FAKE)

    def call(dims, **kw):
        a = dict(ok_args, **kw)
        return lib.tb_decode_attn(ctypes.byref(dims), a["Q"], a["K"], a["V"], a["ctx"], 0.088, a["out"],
                                  a["ws"], kw.get("ws_bytes", ws_bytes), None)

    assert call(_d(head_dim=96)) == _lib.TB_ERR_UNSUPPORTED
    assert b"head_dim" in lib.tb_last_error()
    assert call(_d(n_q_heads=24)) == _lib.TB_ERR_UNSUPPORTED           # group of 3
    assert call(_d(n_q_heads=30)) == _lib.TB_ERR_INVALID_ARG           # not a multiple
    assert call(d, Q=0) == _lib.TB_ERR_INVALID_ARG
    assert call(d, K=MIS) == _lib.TB_ERR_INVALID_ARG
    assert call(d, ws_bytes=ws_bytes - 1) == _lib.TB_ERR_WORKSPACE
    assert call(_d(batch=0)) == _lib.TB_ERR_INVALID_ARG
    assert call(_d(batch=65536)) == _lib.TB_ERR_UNSUPPORTED           # a grid dimension limit
    assert b"65535" in lib.tb_last_error()
    assert lib.tb_attn_workspace_bytes(ctypes.byref(_d(batch=65536))) == 0
    st = lib.tb_sparse_decode_attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 16, 0, FAKE, 0.088, FAKE, FAKE,
                                   ws_bytes, None)
    assert st == _lib.TB_ERR_INVALID_ARG and b"window" in lib.tb_last_error()
    st = lib.tb_sparse_decode_attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 16, 64, 0, 0.088, FAKE, FAKE,
                                   ws_bytes, None)
    assert st == _lib.TB_ERR_INVALID_ARG


def test_plan_and_planned_attention_reject_bad_arguments(lib):
    d = _d()
    ws_bytes = lib.tb_attn_workspace_bytes(ctypes.byref(d))
    plan = lambda **kw: lib.tb_attn_plan(ctypes.byref(kw.get("d", d)), kw.get("bits", FAKE), kw.get("ctx", FAKE),  # noqa: E731
                                         kw.get("sink", 16), kw.get("window", 64), kw.get("plan", FAKE),
                                         kw.get("ws", FAKE), kw.get("ws_bytes", 256), None)
    assert plan(bits=0) == _lib.TB_ERR_INVALID_ARG
    assert plan(plan=FAKE + 2) == _lib.TB_ERR_INVALID_ARG  # int32 entries: 4-byte alignment
    assert plan(window=0) == _lib.TB_ERR_INVALID_ARG and b"window" in lib.tb_last_error()
    assert plan(sink=-1) == _lib.TB_ERR_INVALID_ARG
    assert plan(ws_bytes=255) == _lib.TB_ERR_WORKSPACE
    assert plan(d=_d(head_dim=96)) == _lib.TB_ERR_UNSUPPORTED
    st = lib.tb_sparse_decode_attn_planned(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 16, 64, FAKE, 0, 0.088, FAKE,
                                           FAKE, ws_bytes, None)
    assert st == _lib.TB_ERR_INVALID_ARG and b"plan" in lib.tb_last_error()
    st = lib.tb_sparse_decode_attn_planned(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 16, 0, FAKE, FAKE, 0.088,
                                           FAKE, FAKE, ws_bytes, None)
    assert st == _lib.TB_ERR_INVALID_ARG and b"window" in lib.tb_last_error()


def test_select_rejects_bad_arguments(lib):
    d = _d()
    wsb = lib.tb_score_select_workspace_bytes(ctypes.byref(d))

    def call(dims=d, stride=32 * 32, sink=16, window=64, budget=8192, nbr=1, idx_cap=3 * 8192, ws_bytes=wsb):
        return lib.tb_score_select(ctypes.byref(dims), FAKE, stride, FAKE, FAKE, sink, window, budget, nbr, FAKE,
                                   idx_cap, FAKE, FAKE, FAKE, ws_bytes, None)

    assert call(idx_cap=3 * 8192 - 1) == _lib.TB_ERR_INVALID_ARG
    assert b"idx_cap" in lib.tb_last_error()
    assert call(nbr=17) == _lib.TB_ERR_INVALID_ARG
    assert call(budget=0) == _lib.TB_ERR_INVALID_ARG
    assert call(sink=-1) == _lib.TB_ERR_INVALID_ARG
    assert call(stride=31 * 32) == _lib.TB_ERR_INVALID_ARG
    assert call(dims=_d(d_proj=8)) == _lib.TB_ERR_UNSUPPORTED
    assert call(ws_bytes=wsb // 2) == _lib.TB_ERR_WORKSPACE
    # small contexts: idx_cap may be ctx_cap when that is below (2*nbr+1)*budget
    small = _d(ctx_cap=300)
    w2 = lib.tb_score_select_workspace_bytes(ctypes.byref(small))
    st = lib.tb_score_select(ctypes.byref(small), FAKE, 32 * 32, FAKE, FAKE, 4, 16, 8192, 1, FAKE, 299,
                             FAKE, FAKE, FAKE, w2, None)
    assert st == _lib.TB_ERR_INVALID_ARG


def test_select_group_rejects_bad_arguments(lib):
    d = _d()
    wsb = lib.tb_score_select_workspace_bytes(ctypes.byref(d))

    def call(reduce=0, qp=FAKE, idx_cap=3 * 8192):
        return lib.tb_score_select_group(ctypes.byref(d), qp, 32 * 32, FAKE, FAKE, 16, 64, 8192, 1, reduce, FAKE,
                                         idx_cap, FAKE, FAKE, FAKE, wsb, None)

    assert call(reduce=2) == _lib.TB_ERR_INVALID_ARG
    assert b"reduce" in lib.tb_last_error()
    assert call(reduce=-1) == _lib.TB_ERR_INVALID_ARG
    # a valid reduce goes through the same checks as tb_score_select
    assert call(qp=0) == _lib.TB_ERR_INVALID_ARG
    assert b"tb_score_select_group" in lib.tb_last_error() and b"qp" in lib.tb_last_error()
    assert call(reduce=1, idx_cap=3 * 8192 - 1) == _lib.TB_ERR_INVALID_ARG


def test_select_inclusive_rejects_bad_arguments(lib):
    d = _d()
    wsb = lib.tb_score_select_workspace_bytes(ctypes.byref(d))

    def call(budget=8192, idx_cap=8192):
        return lib.tb_score_select_inclusive(ctypes.byref(d), FAKE, 32 * 32, FAKE, FAKE, 16, 64, budget, 1, FAKE,
                                             idx_cap, FAKE, FAKE, FAKE, wsb, None)

    assert call(budget=8193, idx_cap=8193) == _lib.TB_ERR_UNSUPPORTED
    assert call(idx_cap=8191) == _lib.TB_ERR_INVALID_ARG
    assert b"idx_cap" in lib.tb_last_error() and b"tb_score_select_inclusive" in lib.tb_last_error()


def test_kv_append_rejects_bad_arguments(lib):
    d = _d()

    def call(n_layers=32, src=FAKE, caches=FAKE, ctx=FAKE, ws=FAKE, ws_bytes=256):
        return lib.tb_kv_append(ctypes.byref(d), n_layers, src, caches, ctx, ws, ws_bytes, None)

    assert call(n_layers=0) == _lib.TB_ERR_INVALID_ARG
    assert call(caches=0) == _lib.TB_ERR_INVALID_ARG
    assert b"caches" in lib.tb_last_error()
    assert call(caches=FAKE + 4) == _lib.TB_ERR_INVALID_ARG
    assert call(src=FAKE + 8) == _lib.TB_ERR_INVALID_ARG
    assert call(ws_bytes=255) == _lib.TB_ERR_WORKSPACE


def test_selftest_rejects_bad_arguments(lib):
    assert lib.tb_selftest_bounded_wait(FAKE, 256, 0, None) == _lib.TB_ERR_INVALID_ARG
    assert lib.tb_selftest_bounded_wait(FAKE, 255, 1000, None) == _lib.TB_ERR_WORKSPACE
    assert lib.tb_selftest_bounded_wait(0, 256, 1000, None) == _lib.TB_ERR_INVALID_ARG


def test_predict_and_project_reject_bad_arguments(lib):
    wsb = lib.tb_predict_queries_workspace_bytes(1, 4096, 1024, 4096)
    assert lib.tb_predict_queries(FAKE, FAKE, FAKE, FAKE, 17, 4096, 1024, 4096, FAKE, wsb, None) == \
        _lib.TB_ERR_UNSUPPORTED
    assert lib.tb_predict_queries(FAKE, FAKE, FAKE, FAKE, 1, 4000, 1024, 4096, FAKE, wsb, None) == \
        _lib.TB_ERR_UNSUPPORTED
    assert lib.tb_predict_queries(FAKE, MIS, FAKE, FAKE, 1, 4096, 1024, 4096, FAKE, wsb, None) == \
        _lib.TB_ERR_INVALID_ARG
    assert lib.tb_predict_queries(FAKE, FAKE, FAKE, FAKE, 1, 4096, 1024, 4096, FAKE, wsb - 1, None) == \
        _lib.TB_ERR_WORKSPACE
    d = _d()
    assert lib.tb_project_keys(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, -1, FAKE, 256, None) == \
        _lib.TB_ERR_INVALID_ARG
    assert lib.tb_project_keys(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, 256, None) == _lib.TB_OK
    assert lib.tb_project_keys(ctypes.byref(_d(d_proj=64)), FAKE, FAKE, FAKE, FAKE, FAKE, 64, FAKE, 256, None) \
        == _lib.TB_ERR_UNSUPPORTED


def test_binding_refuses_host_tensors(lib):
    d = _d(ctx_cap=128)
    t = torch.zeros(16, dtype=torch.bfloat16)
    with pytest.raises(_lib.TbError):
        _lib.decode_attn(d, t, t, t, torch.zeros(1, dtype=torch.int32), 0.1, torch.zeros(4), t)


def test_binding_refuses_another_abi_version(lib, monkeypatch):
    monkeypatch.setattr(_lib, "TB_ABI_VERSION", _lib.TB_ABI_VERSION - 1)
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(_lib.TbError, match="ABI version"):
        _lib.load()
    assert _lib._lib is None            # nothing cached from the refused load


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "tb.h"
int main(void) {
    tb_dims d = {1, 32, 8, 96, 32, 4096};
    if (tb_abi_version() != TB_ABI_VERSION) return 1;
    if (strcmp(tb_status_str(TB_ERR_WORKSPACE), "TB_ERR_WORKSPACE") != 0) return 2;
    if (tb_attn_workspace_bytes(&d) != 0) return 3;           /* head_dim 96 is not built */
    d.head_dim = 128;
    if (tb_attn_workspace_bytes(&d) == 0) return 4;
    if (tb_decode_attn(&d, NULL, NULL, NULL, NULL, 0.1f, NULL, NULL, 0, NULL) != TB_ERR_INVALID_ARG) return 5;
    printf("%s\n", tb_last_error());
    return 0;
}
"""


def test_header_is_plain_c_and_the_library_links_from_c(lib, tmp_path):
    # the boundary is a C ABI: tb.h compiles as strict C99 and a C program
    # links against libtb.so and gets host-side validation without a GPU
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "main.c"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "main"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-L", libdir, "-ltb", f"-Wl,-rpath,{libdir}",
                    "-o", str(exe)], check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, (res.returncode, res.stdout, res.stderr)
    assert "16-byte aligned" in res.stdout


def test_score_export_rejects_bad_arguments(lib):
    d = _d()
    wsb = lib.tb_score_select_workspace_bytes(ctypes.byref(d))
    call = lambda dims, ws=FAKE, nb=wsb, ctx=FAKE, sink=16, window=64, out=FAKE: lib.tb_score_select_scores(  # noqa: E731
        ctypes.byref(dims), ws, nb, ctx, sink, window, out, None)
    assert call(_d(d_proj=24)) == _lib.TB_ERR_UNSUPPORTED
    assert call(d, nb=wsb - 1) == _lib.TB_ERR_WORKSPACE
    assert call(d, out=0) == _lib.TB_ERR_INVALID_ARG
    assert call(d, ctx=FAKE + 2) == _lib.TB_ERR_INVALID_ARG
    assert call(d, window=0) == _lib.TB_ERR_INVALID_ARG
    assert call(_d(ctx_cap=(1 << 19) + 1)) == _lib.TB_ERR_UNSUPPORTED


def test_noalloc_accepts_exactly_the_workspace_entry_points_dims(lib):
    # both sparse entry points run the same host checks; the no-alloc one then
    # also bounds the scratch the dims need
    def noalloc(dims, **kw):
        a = dict(Q=FAKE, K=FAKE, V=FAKE, ctx=FAKE, sink=16, window=64, bits=FAKE, scale=0.088, out=FAKE)
        a.update(kw)
        return lib.tb_sparse_decode_attn_noalloc(ctypes.byref(dims), a["Q"], a["K"], a["V"], a["ctx"], a["sink"],
                                                 a["window"], a["bits"], a["scale"], a["out"], None)

    def with_ws(dims, **kw):
        a = dict(Q=FAKE, K=FAKE, V=FAKE, ctx=FAKE, sink=16, window=64, bits=FAKE, scale=0.088, out=FAKE)
        a.update(kw)
        nb = lib.tb_attn_workspace_bytes(ctypes.byref(_d())) or 256
        return lib.tb_sparse_decode_attn(ctypes.byref(dims), a["Q"], a["K"], a["V"], a["ctx"], a["sink"],
                                         a["window"], a["bits"], a["scale"], a["out"], FAKE, nb, None)

    cases = [(_d(ctx_cap=(1 << 22) + 1), {}), (_d(head_dim=96), {}), (_d(n_q_heads=24), {}),
             (_d(batch=65536), {}), (_d(), dict(Q=MIS)), (_d(), dict(bits=0)), (_d(), dict(window=0)),
             (_d(), dict(sink=-1)), (_d(), dict(scale=float("inf")))]
    for dims, kw in cases:
        want = with_ws(dims, **kw)
        assert want in (_lib.TB_ERR_INVALID_ARG, _lib.TB_ERR_UNSUPPORTED), (dims.ctx_cap, kw)
        assert noalloc(dims, **kw) == want, (dims.ctx_cap, kw)
    # valid dims beyond the fixed scratch: rejected before any CUDA call
    assert noalloc(_d(batch=16, ctx_cap=32896)) == _lib.TB_ERR_WORKSPACE


def test_attention_launch_mode_is_per_thread_and_checked(lib):
    import threading
    assert lib.tb_attn_launch_mode() == _lib.TB_ATTN_WAIT_ALL
    assert lib.tb_attn_set_launch_mode(7) == _lib.TB_ERR_INVALID_ARG
    assert lib.tb_attn_set_launch_mode(_lib.TB_ATTN_PREFETCH_KV) == _lib.TB_OK
    seen = []
    t = threading.Thread(target=lambda: seen.append(lib.tb_attn_launch_mode()))
    t.start()
    t.join()
    assert seen == [_lib.TB_ATTN_WAIT_ALL], "another thread keeps the default"
    assert lib.tb_attn_launch_mode() == _lib.TB_ATTN_PREFETCH_KV
    assert lib.tb_attn_set_launch_mode(_lib.TB_ATTN_WAIT_ALL) == _lib.TB_OK


def test_context_parallel_calls_reject_bad_arguments(lib):
    d = _d()
    wsb = lib.tb_score_select_workspace_bytes(ctypes.byref(d))
    # export: misaligned candidates, bad budget, offset overflow, short workspace
    exp = lambda dims=d, ws=FAKE, nb=wsb, idx=FAKE, cap=8192, cnt=FAKE, budget=8192, off=0, cand=FAKE: \
        lib.tb_select_export_candidates(ctypes.byref(dims), ws, nb, idx, cap, cnt, budget, off, cand, None)  # noqa: E731
    assert exp(cand=FAKE + 4) == _lib.TB_ERR_INVALID_ARG
    assert exp(budget=0) == _lib.TB_ERR_INVALID_ARG
    assert exp(off=-1) == _lib.TB_ERR_INVALID_ARG
    assert exp(off=0x7fffffff) == _lib.TB_ERR_INVALID_ARG
    assert exp(nb=wsb - 1) == _lib.TB_ERR_WORKSPACE
    assert exp(dims=_d(d_proj=24)) == _lib.TB_ERR_UNSUPPORTED

    def merge(**kw):
        a = dict(dims=d, cand=FAKE, ranks=4, budget=8192, ctx=FAKE, sink=16, window=64, nbr=1, idx=FAKE,
                 cap=24576, cnt=FAKE, sb=0, sl=16384, lcap=16448, bits=FAKE, ws=FAKE, nb=256)
        a.update(kw)
        return lib.tb_select_merge_candidates(ctypes.byref(a["dims"]), a["cand"], a["ranks"], a["budget"], a["ctx"],
                                              a["sink"], a["window"], a["nbr"], a["idx"], a["cap"], a["cnt"], a["sb"],
                                              a["sl"], a["lcap"], a["bits"], a["ws"], a["nb"], None)
    assert merge(sb=16) == _lib.TB_ERR_INVALID_ARG            # shard_begin not a multiple of 32
    assert merge(sl=20000) == _lib.TB_ERR_INVALID_ARG         # shard longer than its local capacity
    assert merge(sb=65536, sl=16384, lcap=16448) == _lib.TB_ERR_INVALID_ARG   # past ctx_cap
    assert merge(ranks=0) == _lib.TB_ERR_INVALID_ARG
    assert merge(cap=100) == _lib.TB_ERR_INVALID_ARG          # idx_cap below the largest selection
    assert merge(window=0) == _lib.TB_ERR_INVALID_ARG
    assert merge(nb=255) == _lib.TB_ERR_WORKSPACE
    assert merge(cand=FAKE + 4) == _lib.TB_ERR_INVALID_ARG
    # partial attention and combine
    ab = lib.tb_attn_workspace_bytes(ctypes.byref(d))
    part = lambda dims=d, bits=FAKE, nb=ab, scale=0.088: lib.tb_sparse_decode_attn_partial(  # noqa: E731
        ctypes.byref(dims), FAKE, FAKE, FAKE, FAKE, bits, scale, FAKE, FAKE, nb, None)
    assert part(bits=0) == _lib.TB_ERR_INVALID_ARG
    assert part(nb=ab - 1) == _lib.TB_ERR_WORKSPACE
    assert part(dims=_d(head_dim=96)) == _lib.TB_ERR_UNSUPPORTED
    assert part(scale=float("nan")) == _lib.TB_ERR_INVALID_ARG
    assert lib.tb_attn_combine(FAKE, 0, 1, 32, 128, FAKE, None) == _lib.TB_ERR_INVALID_ARG
    assert lib.tb_attn_combine(FAKE, 2, 1, 32, 96, FAKE, None) == _lib.TB_ERR_UNSUPPORTED
    assert lib.tb_attn_combine(FAKE + 2, 2, 1, 32, 128, FAKE, None) == _lib.TB_ERR_INVALID_ARG
