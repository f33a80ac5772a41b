"""CPU-side checks of the C ABI: the library loads, exports every entry point
include/fbk.h declares, and rejects bad arguments on the host before any CUDA
call (nothing here launches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fbk():
    from cached_block_attention_b200 import build
    build.build()
    from cached_block_attention_b200 import fbk as m
    return m


def declared_entry_points(header="fbk.h"):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fbk_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(fbk):
    names = declared_entry_points()
    assert len(names) >= 7
    for n in names:
        assert hasattr(fbk.lib, n), n
    assert set(fbk.EXPORTS) == set(names)


def test_test_build_exports_its_hooks_and_the_library_does_not(fbk):
    """libfbk_testhooks.so exports every fbk.h entry point plus the hooks of
    include/fbk_test_hooks.h; the library proper has none."""
    from cached_block_attention_b200 import build
    hooks = ctypes.CDLL(build.TEST_LIB)
    hook_names = declared_entry_points("fbk_test_hooks.h")
    assert hook_names == ["fbk_test_fp8_group_scale", "fbk_test_set_wait_fault"]
    for n in declared_entry_points() + hook_names:
        assert hasattr(hooks, n), n
    for n in hook_names:
        assert not hasattr(fbk.lib, n), n


def test_status_strings(fbk):
    for code in (0, -1, -2, -3, -4, -5):
        assert fbk.status_string(code) not in ("", "unknown status")
    assert fbk.status_string(7) == "unknown status"


def _shape(fbk, **kw):
    s = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, block_len=32,
             softmax_scale=1.0, rope_base=1e4, mode=0)
    s.update(kw)
    return fbk.CShape(**s)


def _cache(fbk, **kw):
    c = dict(k=0x10000, v=0x20000, paged=0, page_size=0, max_pages_per_seq=0,
             capacity_tokens=1024, num_pages=0, page_table=None, prefix_lens=0x30000,
             error_flags=None)
    c.update(kw)
    return fbk.CCache(**c)


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), -1), (dict(n_q_heads=0), -1), (dict(block_len=0), -1), (dict(mode=3), -1),
    (dict(rope_base=-1.0), -1), (dict(softmax_scale=float("nan")), -1), (dict(softmax_scale=0.0), -1),
    (dict(softmax_scale=-0.5), -1),
    (dict(head_dim=96), -2), (dict(n_q_heads=6, n_kv_heads=4), -2), (dict(block_len=65), -2),
    (dict(n_q_heads=16, n_kv_heads=2, block_len=64), -2), (dict(batch=1025), -2),
])
def test_shape_validation(fbk, kw, code):
    s = _shape(fbk, **kw)
    c = _cache(fbk)
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    st = fbk.lib.fbk_prefix_partial(ctypes.byref(s), ctypes.c_void_p(0x70000), ctypes.byref(c),
                                    ctypes.byref(p), ctypes.c_void_p(0x80000), 1 << 30, 4, None)
    assert st == code
    st = fbk.lib.fbk_block_attn_merge(ctypes.byref(s), ctypes.c_void_p(0x70000), ctypes.c_void_p(0x70000),
                                      ctypes.c_void_p(0x70000), ctypes.c_void_p(0x30000), ctypes.byref(p),
                                      ctypes.c_void_p(0x90000), None, None)
    assert st == code
    if kw != dict(block_len=65):  # B in (64, 256] with G*B <= 256 is a valid prefix shape (fbk_prefix_partial_at)
        assert fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(s), ctypes.byref(c), 4) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), -1), (dict(prefix_lens=None), -1), (dict(capacity_tokens=0), -1),
    (dict(k=0x10008), -2),
    (dict(paged=1, page_size=64, max_pages_per_seq=4, num_pages=8, page_table=None), -1),
    (dict(paged=1, page_size=48, max_pages_per_seq=4, num_pages=8, page_table=0x1000), -2),
    (dict(paged=1, page_size=8, max_pages_per_seq=4, num_pages=8, page_table=0x1000), -2),
    (dict(capacity_tokens=1 << 31), -3),
])
def test_cache_validation(fbk, kw, code):
    s = _shape(fbk)
    c = _cache(fbk, **kw)
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    st = fbk.lib.fbk_prefix_partial(ctypes.byref(s), ctypes.c_void_p(0x70000), ctypes.byref(c),
                                    ctypes.byref(p), ctypes.c_void_p(0x80000), 1 << 30, 4, None)
    assert st == code
    st = fbk.lib.fbk_commit_block_rope_append(ctypes.byref(s), ctypes.c_void_p(0x70000),
                                              ctypes.c_void_p(0x70000), ctypes.byref(c), None)
    assert st == code
    st = fbk.lib.fbk_full_ref_attn(ctypes.byref(s), ctypes.c_void_p(0x70000), ctypes.c_void_p(0x70000),
                                   ctypes.c_void_p(0x70000), ctypes.byref(c), ctypes.c_void_p(0x90000),
                                   None, None)
    assert st == code


def test_null_pointers(fbk):
    s = _shape(fbk)
    c = _cache(fbk)
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    assert fbk.lib.fbk_prefix_partial(None, None, None, None, None, 0, 0, None) == -1
    assert fbk.lib.fbk_prefix_partial(ctypes.byref(s), None, ctypes.byref(c), ctypes.byref(p),
                                      ctypes.c_void_p(0x80000), 1 << 30, 4, None) == -1
    bad = fbk.CPartial(0x40000, None, 0x60000)
    assert fbk.lib.fbk_prefix_partial(ctypes.byref(s), ctypes.c_void_p(0x70000), ctypes.byref(c),
                                      ctypes.byref(bad), ctypes.c_void_p(0x80000), 1 << 30, 4, None) == -1
    assert fbk.lib.fbk_block_attn_merge(ctypes.byref(s), None, None, None, None, None, None, None, None) == -1


def test_workspace_size_and_check(fbk):
    s = _shape(fbk)  # G*B = 64 rows, d = 128, b*Hkv = 2 units
    c = _cache(fbk)
    n = fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(s), ctypes.byref(c), 10)
    slots = 10 + 2
    states = slots * 64 * 130 * 4            # O~, m, l per slot and row (fp32)
    qrot = 2 * 128 * 128 * 2                 # rotated queries: units x one 128-row M-tile x d (bf16)
    assert n >= states + qrot
    assert n < states + qrot + 4 * 256
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    st = fbk.lib.fbk_prefix_partial(ctypes.byref(s), ctypes.c_void_p(0x70000), ctypes.byref(c),
                                    ctypes.byref(p), ctypes.c_void_p(0x80000), n - 1, 10, None)
    assert st == -4
    st = fbk.lib.fbk_prefix_partial(ctypes.byref(s), ctypes.c_void_p(0x70000), ctypes.byref(c),
                                    ctypes.byref(p), None, n, 10, None)
    assert st == -4
    assert fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(s), ctypes.byref(c), -1) == 0


@pytest.mark.parametrize("name", ["tiny", "llada8b", "dream7b_gqa", "long131k", "ragged_paged"])
def test_static_scratch_covers_every_workload(fbk, name):
    """The built-in 32 MiB scratch of fbk_prefix_partial_static_scratch holds the
    workspace of every workload shape at one share per SM of a B200 (148)."""
    from cached_block_attention_b200 import synth
    wl = synth.WORKLOADS[name]
    s = fbk.CShape(batch=wl.batch, n_q_heads=wl.n_q_heads, n_kv_heads=wl.n_kv_heads,
                   head_dim=wl.head_dim, block_len=wl.block_len, softmax_scale=1.0,
                   rope_base=wl.rope_base, mode=0)
    n = fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(s), None, 148)
    rows = wl.n_q_heads // wl.n_kv_heads * wl.block_len
    units = wl.batch * wl.n_kv_heads
    assert n >= (148 + units) * rows * (wl.head_dim + 2) * 4 + units * 128 * ((rows + 127) // 128) * wl.head_dim * 2
    assert n <= fbk.STATIC_SCRATCH_BYTES


def _layer(fbk, lens=0x30000, interval=2, q=0x70000, cache_kw=None):
    c = _cache(fbk, prefix_lens=lens, **(cache_kw or {}))
    return fbk.CLayerBlock(q, 0x71000, 0x72000, c, fbk.CPartial(0x40000, 0x50000, 0x60000), 0x90000, None,
                           interval)


def _decode(fbk, layers, steps=4, commit=1, ws=None, ws_bytes=0, splits=4, shape=None):
    s = shape or _shape(fbk)
    arr = (fbk.CLayerBlock * max(1, len(layers)))(*layers)
    return fbk.lib.fbk_decode_block(ctypes.byref(s), arr if layers else None, len(layers), steps, commit,
                                    ctypes.c_void_p(ws) if ws else None, ws_bytes, splits, None)


def test_decode_block_argument_checks(fbk):
    """fbk_decode_block checks every layer before any launch; a workspace that
    is missing (-4) is the last check, so reaching it means the rest passed."""
    ok = [_layer(fbk, lens=0x30000), _layer(fbk, lens=0x31000, interval=1)]
    assert _decode(fbk, ok) == -4
    assert _decode(fbk, []) == -1                                     # no layers
    assert _decode(fbk, ok, steps=0) == -1
    assert _decode(fbk, ok, splits=-1) == -1
    assert _decode(fbk, ok, shape=_shape(fbk, head_dim=96)) == -2
    assert _decode(fbk, [ok[0], _layer(fbk, lens=0x31000, interval=0)]) == -1
    assert _decode(fbk, [ok[0], _layer(fbk, lens=0x31000, cache_kw=dict(k=None))]) == -1
    assert _decode(fbk, [ok[0], _layer(fbk, lens=0x31000, q=0x70008)]) == -2
    bad_prefix = _layer(fbk, lens=0x31000)
    bad_prefix.prefix = fbk.CPartial(0x40000, None, 0x60000)
    assert _decode(fbk, [ok[0], bad_prefix]) == -1
    # a shared length array is refused only when the layers commit
    shared = [_layer(fbk, lens=0x30000), _layer(fbk, lens=0x30000)]
    assert _decode(fbk, shared, commit=1) == -1
    assert _decode(fbk, shared, commit=0) == -4
    n = fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(_shape(fbk)), None, 4)
    assert _decode(fbk, ok, ws=0x100000, ws_bytes=n - 1) == -4
    assert _decode(fbk, ok, ws=0x100010, ws_bytes=n) == -2          # workspace not 256-byte aligned


def test_decode_block_adaptive_argument_checks(fbk):
    """fbk_decode_block_adaptive: the policy is checked with the layers, before
    any launch; a missing workspace (-4) is the last check."""
    ok = [_layer(fbk, lens=0x30000), _layer(fbk, lens=0x31000, interval=0)]  # intervals are ignored
    pol = fbk.CDriftPolicy(0.1, 0x80000, 0x81000, 0x82000, 0x83000)

    def call(layers=ok, policy=pol, steps=4, shape=None):
        s = shape or _shape(fbk)
        arr = (fbk.CLayerBlock * max(1, len(layers)))(*layers)
        return fbk.lib.fbk_decode_block_adaptive(ctypes.byref(s), arr if layers else None, len(layers), steps, 1,
                                                 ctypes.byref(policy) if policy else None, None, 0, 4, None)

    assert call() == -4
    assert call(policy=None) == -1
    assert call(layers=[]) == -1
    assert call(steps=0) == -1
    for theta in (-1.0, float("nan")):
        assert call(policy=fbk.CDriftPolicy(theta, 0x80000, 0x81000, 0x82000, 0x83000)) == -1
    assert call(policy=fbk.CDriftPolicy(float("inf"), 0x80000, 0x81000, 0x82000, 0x83000)) == -4
    assert call(policy=fbk.CDriftPolicy(0.1, None, 0x81000, 0x82000, 0x83000)) == -1
    assert call(policy=fbk.CDriftPolicy(0.1, 0x80000, 0x81000, 0x82000, None)) == -1
    assert call(shape=_shape(fbk, mode=1)) == -2  # the adaptive refresh runs on the bf16 path


def test_fp8_group_quant_argument_checks(fbk):
    """Host checks of fbk_fp8_group_quant; none of these reach a CUDA call."""
    q = fbk.lib.fbk_fp8_group_quant
    x, c, s = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    assert q(x, 4, 100, c, s, None) == -1                   # cols not a multiple of 128
    assert q(x, -1, 128, c, s, None) == -1
    assert q(x, 4, -128, c, s, None) == -1
    assert q(None, 0, 128, None, None, None) == 0           # empty: nothing enqueued
    assert q(None, 4, 0, None, None, None) == 0
    assert q(None, 4, 128, c, s, None) == -1
    assert q(x, 4, 128, None, s, None) == -1
    assert q(x, 4, 128, c, None, None) == -1
    assert q(ctypes.c_void_p(0x10008), 4, 128, c, s, None) == -2   # x not 16-byte aligned
    assert q(x, 4, 128, ctypes.c_void_p(0x20004), s, None) == -2   # codes not 8-byte aligned
    assert q(x, 4, 128, c, ctypes.c_void_p(0x30002), None) == -2   # scales not 4-byte aligned
    assert q(x, 1 << 33, 1 << 8, c, s, None) == -3          # more than 2^40 elements


def test_facache_unchanged_rows_argument_checks(fbk):
    """Host checks of fbk_facache_unchanged_rows; none of these reach a CUDA call."""
    f = fbk.lib.fbk_facache_unchanged_rows
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    ptr = ctypes.c_void_p
    args = lambda **kw: dict(dict(q=ptr(0x70000), k=ptr(0x71000), v=ptr(0x72000), pos=ptr(0x30000),
                                  out=ptr(0x90000)), **kw)

    def call(shape=None, n=100, part=p, **kw):
        a = args(**kw)
        s = shape or _shape(fbk)
        return f(ctypes.byref(s), n, a["q"], ctypes.byref(part) if part is not None else None, a["k"], a["v"],
                 a["pos"], a["out"], None, None)
    assert call(shape=_shape(fbk, mode=1)) == -2           # bf16 mode only
    assert call(shape=_shape(fbk, head_dim=96)) == -2
    assert call(n=-1) == -1
    assert call(n=0, q=None, part=None) == 0               # no rows: nothing enqueued
    assert call(q=None) == -1
    assert call(pos=None) == -1
    assert call(part=fbk.CPartial(0x40000, None, 0x60000)) == -1
    assert call(q=ptr(0x70008)) == -2
    assert call(part=fbk.CPartial(0x40008, 0x50000, 0x60000)) == -2
    assert call(n=1 << 30, shape=_shape(fbk, batch=4)) == -3
    # the block path's G*B <= 256 limit does not apply (its rows are U's), B <= 64 does
    assert call(n=1 << 30, shape=_shape(fbk, n_q_heads=16, n_kv_heads=1, block_len=64)) == -3
    assert call(shape=_shape(fbk, block_len=65)) == -2


def test_plain_c_host_builds_and_calls_the_library(fbk, tmp_path):
    """A C99 program includes include/fbk.h, links libfbk.so and calls entry
    points that answer on the host (status strings, workspace sizes, argument
    errors): the boundary needs no C++, Python or torch."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "host.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "fbk.h"
int main(void) {
  fbk_shape s = {1, 4, 2, 128, 32, 1.0f, 10000.0, FBK_BF16};
  fbk_kv_cache c;
  memset(&c, 0, sizeof c);
  if (strcmp(fbk_status_string(FBK_ERR_WORKSPACE), "workspace missing or too small") != 0) return 1;
  if (fbk_prefix_workspace_bytes(&s, &c, 10) == 0) return 2;
  s.head_dim = 96;
  if (fbk_prefix_workspace_bytes(&s, &c, 10) != 0) return 3;
  if (fbk_prefix_partial(&s, NULL, &c, NULL, NULL, 0, 4, NULL) != FBK_ERR_UNSUPPORTED) return 4;
  s.head_dim = 128;
  if (fbk_prefix_partial(&s, NULL, &c, NULL, NULL, 0, 4, NULL) != FBK_ERR_INVALID_ARG) return 5;
  if (fbk_fp8_group_quant(NULL, 4, 100, NULL, NULL, NULL) != FBK_ERR_INVALID_ARG) return 6;
  puts("ok");
  return 0;
}
''')
    lib_dir = os.path.dirname(fbk.LIB_PATH)
    exe = tmp_path / "host"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", f"-I{ROOT}/include",
                        str(src), f"-L{lib_dir}", "-lfbk", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)

def test_prefix_partial_at_argument_checks(fbk):
    """fbk_prefix_partial_at: q_pos is required; blocks longer than 64 are accepted while G*B <= 256."""
    c = _cache(fbk)
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    f = fbk.lib.fbk_prefix_partial_at
    q, pos, ws = ctypes.c_void_p(0x70000), ctypes.c_void_p(0x30000), ctypes.c_void_p(0x80000)
    s = _shape(fbk, n_q_heads=2, n_kv_heads=2, block_len=256)           # G*B = 256
    assert f(ctypes.byref(s), q, None, ctypes.byref(c), ctypes.byref(p), ws, 1 << 30, 4, None) == -1
    assert f(ctypes.byref(s), q, pos, ctypes.byref(c), ctypes.byref(p), None, 0, 4, None) == -4
    s2 = _shape(fbk, n_q_heads=4, n_kv_heads=2, block_len=129)          # G*B = 258
    assert f(ctypes.byref(s2), q, pos, ctypes.byref(c), ctypes.byref(p), ws, 1 << 30, 4, None) == -2
    assert fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(s), ctypes.byref(c), 4) > 0


def test_facache_refresh_and_step_argument_checks(fbk):
    """Host checks of fbk_facache_refresh and fbk_facache_step; none reach a CUDA call."""
    s = _shape(fbk)
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    ptr = ctypes.c_void_p
    pos = (ctypes.c_int32 * 1)(10)
    bad_pos = (ctypes.c_int32 * 1)(101)
    c = _cache(fbk)
    paged = _cache(fbk, paged=1, page_size=64, max_pages_per_seq=4, num_pages=8, page_table=0x1000)
    r = fbk.lib.fbk_facache_refresh
    assert r(ctypes.byref(s), 100, ptr(0x70000), pos, ctypes.byref(paged), ctypes.byref(p), None, 0, 4, None) == -2
    assert r(ctypes.byref(s), 100, ptr(0x70000), bad_pos, ctypes.byref(c), ctypes.byref(p), None, 0, 4, None) == -1
    assert r(ctypes.byref(s), 100, ptr(0x70000), None, ctypes.byref(c), ctypes.byref(p), None, 0, 4, None) == -1
    assert r(ctypes.byref(s), 0, None, pos, ctypes.byref(c), None, None, 0, 4, None) == 0
    assert r(ctypes.byref(s), 100, ptr(0x70000), pos, ctypes.byref(c), ctypes.byref(p), None, 0, 4, None) == -4
    n = fbk.lib.fbk_facache_workspace_bytes(ctypes.byref(s), 100, 4)
    assert n > fbk.lib.fbk_prefix_workspace_bytes(ctypes.byref(s), None, 4)
    st = fbk.lib.fbk_facache_step
    args = [ptr(0x70000), ctypes.byref(p), ptr(0x71000), ptr(0x72000), ptr(0x73000), ptr(0x30000), ctypes.byref(c),
            ptr(0x90000), None, ptr(0x91000), None]
    assert st(ctypes.byref(_shape(fbk, mode=1)), 100, *args, ptr(0x100000), n, 4, None) == -2
    assert st(ctypes.byref(s), 100, *args, ptr(0x100000), n - 1, 4, None) == -4
    assert st(ctypes.byref(s), 100, *args, ptr(0x100010), n, 4, None) == -2


def test_sparse_argument_checks(fbk):
    """Host checks of the sparse-prefix calls; none reach a CUDA call."""
    s = _shape(fbk)
    ptr = ctypes.c_void_p
    c = _cache(fbk)
    paged = _cache(fbk, paged=1, page_size=64, max_pages_per_seq=4, num_pages=8, page_table=0x1000)
    huge = _cache(fbk, paged=1, page_size=64, max_pages_per_seq=25601, num_pages=8, page_table=0x1000)
    means = ctypes.cast(ctypes.c_void_p(0x200000), ctypes.POINTER(ctypes.c_float))
    odd_means = ctypes.cast(ctypes.c_void_p(0x200004), ctypes.POINTER(ctypes.c_float))
    kept = ctypes.cast(ctypes.c_void_p(0x210000), ctypes.POINTER(ctypes.c_int32))
    lens = ctypes.cast(ctypes.c_void_p(0x220000), ctypes.POINTER(ctypes.c_int32))
    pm = fbk.lib.fbk_page_means
    assert pm(ctypes.byref(s), ctypes.byref(c), means, None) == -2            # contiguous cache
    assert pm(ctypes.byref(s), ctypes.byref(paged), None, None) == -1
    assert fbk.lib.fbk_select_pages_workspace_bytes(ctypes.byref(s), ctypes.byref(c)) == 0
    n = fbk.lib.fbk_select_pages_workspace_bytes(ctypes.byref(s), ctypes.byref(paged))
    # rotated queries fp32 [b, B, Hq, d] and the scores fp32 [b, Hkv, max_pages], each 256-byte aligned
    assert n == 1 * 32 * 4 * 128 * 4 + 256
    sp = fbk.lib.fbk_select_pages
    q, ws = ptr(0x70000), ptr(0x300000)
    assert sp(ctypes.byref(s), q, ctypes.byref(c), means, 2, kept, lens, ws, n, None) == -2
    assert sp(ctypes.byref(s), q, ctypes.byref(paged), means, 0, kept, lens, ws, n, None) == -1
    assert sp(ctypes.byref(s), q, ctypes.byref(paged), None, 2, kept, lens, ws, n, None) == -1
    assert sp(ctypes.byref(s), q, ctypes.byref(paged), odd_means, 2, kept, lens, ws, n, None) == -2
    assert sp(ctypes.byref(s), q, ctypes.byref(huge), means, 2, kept, lens, ws, 1 << 30, None) == -2
    assert sp(ctypes.byref(s), q, ctypes.byref(paged), means, 2, kept, lens, ws, n - 1, None) == -4
    assert sp(ctypes.byref(s), q, ctypes.byref(paged), means, 2, kept, lens, ptr(0x300010), n, None) == -2
    p = fbk.CPartial(0x40000, 0x50000, 0x60000)
    bad = fbk.CPartial(0x40000, None, 0x60000)
    ro = ctypes.cast(ctypes.c_void_p(0x230000), ctypes.POINTER(ctypes.c_float))
    rl = ctypes.cast(ctypes.c_void_p(0x240000), ctypes.POINTER(ctypes.c_float))
    rc, ra = fbk.lib.fbk_residual_capture, fbk.lib.fbk_residual_apply
    assert rc(ctypes.byref(s), ctypes.byref(p), ctypes.byref(bad), ro, rl, None) == -1
    assert rc(ctypes.byref(s), ctypes.byref(p), ctypes.byref(p), None, rl, None) == -1
    assert ra(ctypes.byref(s), ctypes.byref(bad), ro, rl, ctypes.byref(p), None) == -1
    big = _shape(fbk, n_q_heads=4, n_kv_heads=2, block_len=129)            # G*B = 258
    assert rc(ctypes.byref(big), ctypes.byref(p), ctypes.byref(p), ro, rl, None) == -2
