"""The C-ABI library loads, exports every entry point include/kvs.h declares, and
rejects bad arguments on the host (no GPU needed: nothing here launches)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvs():
    from asymmetric_kv_merging_b200 import build
    build.build()
    from asymmetric_kv_merging_b200 import kvs as mod
    return mod


def header_functions():
    with open(os.path.join(ROOT, "include", "kvs.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_0-9]+\s*\*?\s*(kvs_[a-z_0-9]+)\s*\(",
                                 text, re.M)))


def test_every_declared_function_is_exported(kvs):
    names = header_functions()
    assert {"kvs_score_pairs", "kvs_merge_compact", "kvs_decode_attn", "kvs_workspace_size"} <= set(names)
    lib = ctypes.CDLL(kvs.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert set(kvs.EXPORTS) <= set(names)


def test_status_strings(kvs):
    for code in range(7):
        assert kvs.status_str(code)
    assert kvs.status_str(0) == "ok"


def test_workspace_sizes(kvs):
    d = kvs.make_desc(1, 8, 32, 128, 32768, kvs.BF16)
    for op in (kvs.OP_SCORE, kvs.OP_MERGE, kvs.OP_DECODE):
        n = kvs.workspace_size(d, 32, op)
        assert n > 0 and n % 256 == 0
    # alpha_bar alone needs one fp32 per cached row
    assert kvs.workspace_size(d, 32, kvs.OP_SCORE) >= 8 * 32768 * 4
    bad = kvs.make_desc(1, 8, 32, 96, 32768, kvs.BF16)           # head dim 96 not built
    assert kvs.workspace_size(bad, 32, kvs.OP_SCORE) == 0
    assert kvs.workspace_size(kvs.make_desc(1, 8, 24, 128, 64, kvs.BF16), 32, kvs.OP_DECODE) == 0
    assert kvs.workspace_size(d, 32, 7) == 0


FAKE = 1 << 40          # aligned fake device addresses: validation never dereferences


def _fake(i):
    return ctypes.c_void_p(FAKE + i * (1 << 34))


def _score(kvs, desc, **over):
    args = dict(K=_fake(1), V=_fake(2), logn=None, len=_fake(3), cb=_fake(4), n_recent=32,
                Q=_fake(5), W=32, score=_fake(6), w_b=_fake(7), ws=_fake(8), ws_bytes=1 << 40)
    args.update(over)
    return kvs._lib.kvs_score_pairs(ctypes.byref(desc), args["K"], args["V"], args["logn"],
                                    args["len"], args["cb"], args["n_recent"], args["Q"],
                                    args["W"], args["score"], args["w_b"], args["ws"],
                                    args["ws_bytes"], None)


def test_score_pairs_host_validation(kvs):
    d = kvs.make_desc(1, 8, 32, 128, 1024, kvs.BF16)
    assert _score(kvs, d, K=None) == 1                                   # NULL
    assert _score(kvs, d, K=ctypes.c_void_p(FAKE + 8)) == 1              # misaligned
    assert _score(kvs, d, W=0) == 1
    assert _score(kvs, d, n_recent=-1) == 1
    assert _score(kvs, d, W=33) == 2                                     # G*W > 128
    assert _score(kvs, kvs.make_desc(1, 8, 32, 80, 1024, kvs.BF16)) == 2
    assert _score(kvs, kvs.make_desc(1, 8, 32, 128, 1023, kvs.BF16)) == 1  # odd T_cap
    assert _score(kvs, kvs.make_desc(1, 8, 32, 128, 1024, 5)) == 2
    assert _score(kvs, d, ws_bytes=1024) == 4
    assert _score(kvs, d, ws=None) == 4
    assert _score(kvs, d, ws=ctypes.c_void_p(FAKE + 128)) == 4           # not 256-aligned
    assert _score(kvs, d, score=_fake(1)) == 5                           # score over K


def _merge(kvs, desc, **over):
    a = dict(K=_fake(1), V=_fake(2), logn=_fake(9), len=_fake(3), cb=_fake(4), n_recent=32,
             score=_fake(6), w_b=_fake(7), target=_fake(10), scope=0, T_out=desc.T_cap,
             K_out=_fake(11), V_out=_fake(12), ln_out=_fake(13), len_out=_fake(14),
             dsel=None, doff=None, dkm=None, ws=_fake(8), ws_bytes=1 << 40)
    a.update(over)
    return kvs._lib.kvs_merge_compact(
        ctypes.byref(desc), a["K"], a["V"], a["logn"], a["len"], a["cb"], a["n_recent"], a["score"],
        a["w_b"], a["target"], a["scope"], a["T_out"], a["K_out"], a["V_out"], a["ln_out"],
        a["len_out"], a["dsel"], a["doff"], a["dkm"], a["ws"], a["ws_bytes"], None)


def test_merge_compact_host_validation(kvs):
    d = kvs.make_desc(2, 8, 32, 128, 4096, kvs.BF16)
    assert _merge(kvs, d, target=None) == 1
    assert _merge(kvs, d, scope=2) == 1
    assert _merge(kvs, d, T_out=0) == 1
    assert _merge(kvs, d, K_out=_fake(2)) == 5                 # K_out over V
    assert _merge(kvs, d, dsel=_fake(6)) == 5                  # debug output over score
    assert _merge(kvs, d, V_out=_fake(11)) == 5                # two outputs overlap
    # in-place needs every cache buffer in place and a log-count array
    assert _merge(kvs, d, K_out=_fake(1), V_out=_fake(12)) == 5
    assert _merge(kvs, d, K_out=_fake(1), V_out=_fake(2), ln_out=_fake(9), len_out=_fake(3),
                  ws_bytes=16) == 4
    assert _merge(kvs, d, K_out=_fake(1), V_out=_fake(2), logn=None, ln_out=None,
                  len_out=_fake(3)) == 1
    assert _merge(kvs, d, ws_bytes=256) == 4


def test_decode_host_validation(kvs):
    d = kvs.make_desc(1, 8, 32, 128, 4096, kvs.BF16)
    lib = kvs._lib

    def call(**o):
        a = dict(q=_fake(1), K=_fake(2), V=_fake(3), logn=None, len=_fake(4), kn=None, vn=None,
                 out=_fake(5), ws=_fake(6), ws_bytes=1 << 40)
        a.update(o)
        return lib.kvs_decode_attn(ctypes.byref(d), a["q"], a["K"], a["V"], a["logn"], a["len"],
                                   a["kn"], a["vn"], a["out"], a["ws"], a["ws_bytes"], None)

    assert call(q=None) == 1
    assert call(kn=_fake(7)) == 1                               # k_new without v_new
    assert call(out=_fake(2)) == 5                              # output over K
    assert call(ws_bytes=100) == 4


def _prefill(kvs, desc, **over):
    args = dict(K=_fake(1), V=_fake(2), logn=_fake(9), len=_fake(3), L=0, kc=_fake(10),
                vc=_fake(11), n=512, Q=_fake(5), W=32, budget=2048, sink=32, form=0,
                ws=_fake(8), ws_bytes=1 << 40)
    args.update(over)
    out = ctypes.c_int32(-1)
    st = kvs._lib.kvs_prefill_chunk(ctypes.byref(desc), args["K"], args["V"], args["logn"],
                                    args["len"], args["L"], args["kc"], args["vc"], args["n"],
                                    args["Q"], args["W"], args["budget"], args["sink"],
                                    args["form"], ctypes.byref(out), args["ws"],
                                    args["ws_bytes"], None)
    return st, out.value


def test_prefill_chunk_host_validation_and_plan(kvs):
    d = kvs.make_desc(1, 8, 32, 128, 4096, kvs.BF16)
    assert _prefill(kvs, d, logn=None)[0] == 1                         # counts are required
    assert _prefill(kvs, d, form=4)[0] == 1                            # unknown form bits
    assert _prefill(kvs, d, L=3800, n=512)[0] == 1                     # L + n > T_cap
    assert _prefill(kvs, d, W=33)[0] == 2                              # G*W > 128
    big = kvs.make_desc(1, 8, 32, 128, 16384, kvs.BF16)
    assert _prefill(kvs, big, L=8000, n=512)[0] == 2                   # in-place span > 8192
    # budget below what the protected rows allow: refused before anything is launched
    assert _prefill(kvs, d, L=2048, n=512, budget=40)[0] == 3
    assert _prefill(kvs, d, ws_bytes=16)[0] == 4
    assert kvs.workspace_size(d, 32, kvs.OP_PREFILL) > kvs.workspace_size(d, 32, kvs.OP_SCORE)


def test_prefill_chunk_alias_rules(kvs):
    d = kvs.make_desc(1, 8, 32, 128, 4096, kvs.BF16)
    same = _fake(10)
    # k and v chunks may be one buffer (both are read); the cache may not overlap them
    assert _prefill(kvs, d, kc=same, vc=same, L=2048, n=512, budget=40)[0] == 3
    assert _prefill(kvs, d, kc=_fake(1))[0] == 5
    assert _prefill(kvs, d, logn=_fake(2))[0] == 5


def test_score_pairs_form_host_validation(kvs):
    d = kvs.make_desc(1, 8, 32, 128, 1024, kvs.BF16)

    def call(form, **o):
        a = dict(K=_fake(1), V=_fake(2), ws_bytes=1 << 40)
        a.update(o)
        return kvs._lib.kvs_score_pairs_form(ctypes.byref(d), a["K"], a["V"], None, _fake(3),
                                             _fake(4), 32, _fake(5), 32, _fake(6), _fake(7),
                                             form, _fake(8), a["ws_bytes"], None)

    assert call(4) == 1 and call(-1) == 1                      # unknown form bits
    # the per-query window form needs the tensor-core path; without a device to encode
    # tensor maps on, nothing supports it (on a B200 this shape does)
    if not __import__("torch").cuda.is_available():
        assert call(kvs.FORM_PER_QUERY) == 2
    assert call(kvs.FORM_DIAGONAL, K=None) == 1
    assert call(kvs.FORM_DIAGONAL, ws_bytes=256) == 4
    assert call(kvs.FORM_FULL, ws_bytes=256) == 4


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "kvs.h"
int main(void) {
  kvs_cache_desc d = {1, 8, 32, 128, 32768, KVS_BF16};
  size_t ws = kvs_workspace_size(&d, 32, KVS_OP_DECODE);
  int32_t L = -1;
  /* host-checked argument errors launch nothing and need no GPU */
  kvs_status s = kvs_prefill_chunk(&d, 0, 0, 0, 0, 0, 0, 0, 0, 0, 32, 2048, 32,
                                   KVS_FORM_FULL, &L, 0, 0, 0);
  printf("%d %d %d %s %d\n", kvs_version(), (int)(ws > 0), (int)s, kvs_status_str(KVS_OK), (int)L);
  return 0;
}
"""


def test_plain_c_program_links_and_calls_the_library(kvs, tmp_path):
    """A C99 program built with gcc against include/kvs.h and libkvs.so: the boundary is a
    plain C ABI (no C++ or torch types), and host-only calls work without a GPU."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(kvs.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lkvs", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out == ["1", "1", "1", "ok", "-1"]      # version, size > 0, INVALID_ARG, "ok", untouched


def test_plan_rounds_matches_the_round_rule(kvs):
    import sys
    from hypothesis import given, settings, strategies as st
    sys.path.insert(0, ROOT)
    import bench
    assert kvs.plan_rounds(131072, 32768, 32, 32) == [131072, 65568, 32816, 32768]
    assert kvs.plan_rounds(100, 100, 4, 4) == [100]
    with pytest.raises(kvs.KvsError) as e:
        kvs.plan_rounds(100, 10, 32, 32)                       # span too short to get there
    assert e.value.status == 3
    with pytest.raises(kvs.KvsError) as e:
        kvs.plan_rounds(131072, 32768, 32, 32, max_lens=3)      # 4 lengths needed
    assert e.value.status == 1

    @settings(max_examples=200, deadline=None)
    @given(L=st.integers(0, 200000), frac=st.floats(0.0, 1.0), c0=st.integers(0, 64),
           nr=st.integers(0, 64))
    def check(L, frac, c0, nr):
        target = int(L * frac)
        try:
            want = bench.plan_rounds(L, target, c0, nr)
        except ValueError:
            with pytest.raises(kvs.KvsError):
                kvs.plan_rounds(L, target, c0, nr)
            return
        assert kvs.plan_rounds(L, target, c0, nr) == want

    check()
