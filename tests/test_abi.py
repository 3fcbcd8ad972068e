"""The C ABI: the library loads on a CPU-only host, exports every declared symbol,
and rejects bad arguments synchronously, before any launch."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

import paged_kv_cache_349_b200 as pa
from paged_kv_cache_349_b200._lib import SIGNATURES, lib


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_and_binding_agree():
    declared = _declared_functions()
    assert len(declared) >= 20
    assert sorted(SIGNATURES) == declared


def test_every_declared_symbol_is_exported():
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    assert pa.status_string(0) == "PA_OK"
    assert pa.status_string(pa.PA_ERR_OOM) == "PA_ERR_OOM"
    assert pa.status_string(999) == "PA_ERR_UNKNOWN"
    assert pa.version() >= 100


P = ctypes.c_void_p


def _fake(addr=0x10000):
    return P(addr)


def test_decode_argument_errors_need_no_gpu():
    f = lib.pa_decode
    ok_args = dict(out=_fake(), q=_fake(), k=_fake(), v=_fake(), bt=_fake(), maxb=4, lens=_fake(),
                   B=2, maxlen=64, Hq=8, Hkv=2, d=128, bs=16, NB=64, scale=0.1, pt=-1,
                   ws=None, wsb=0, flag=None, stream=None)

    def call(**kw):
        a = dict(ok_args, **kw)
        return f(a["out"], a["q"], a["k"], a["v"], a["bt"], a["maxb"], a["lens"], a["B"], a["maxlen"],
                 a["Hq"], a["Hkv"], a["d"], a["bs"], a["NB"], a["scale"], a["pt"], a["ws"], a["wsb"],
                 a["flag"], a["stream"])

    assert call(B=0) == pa.PA_OK                         # nothing to do, nothing launched
    assert call(d=96) == pa.PA_ERR_UNSUPPORTED
    assert call(bs=12) == pa.PA_ERR_UNSUPPORTED
    assert call(bs=128) == pa.PA_ERR_UNSUPPORTED
    assert call(Hq=6, Hkv=4) == pa.PA_ERR_UNSUPPORTED    # not a whole group
    assert call(Hq=32, Hkv=2) == pa.PA_ERR_UNSUPPORTED   # group of 16
    assert call(q=None) == pa.PA_ERR_INVALID_ARG
    assert call(q=_fake(0x10008)) == pa.PA_ERR_INVALID_ARG  # misaligned
    assert call(pt=24) == pa.PA_ERR_INVALID_ARG          # not a multiple of block_size
    assert call(pt=16, ws=None) == pa.PA_ERR_INVALID_ARG  # split needs a workspace
    assert call(NB=0) == pa.PA_ERR_INVALID_ARG
    assert call(NB=1 << 30) == pa.PA_ERR_UNSUPPORTED     # TMA row coordinate overflow


def test_cache_op_argument_errors_need_no_gpu():
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 0, 8, 2, 16, 128, None, None) == pa.PA_OK
    assert lib.pa_reshape_and_cache(_fake(), _fake(), _fake(), _fake(), None, 3, 8, 2, 16, 128, None,
                                    None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_reshape_and_cache(_fake(), _fake(), _fake(), _fake(), _fake(), 3, 8, 2, 16, 80, None,
                                    None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_copy_blocks(None, None, None, 0, 8, 2, 16, 128, None, None) == pa.PA_OK
    assert lib.pa_copy_blocks(_fake(), _fake(), None, 2, 8, 2, 16, 128, None, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(_fake(0x10004), _fake(), _fake(), 2, 8, 2, 16, 128, None,
                              None) == pa.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("pt,maxlen,parts", [(512, 32768, 64), (512, 512, 0), (16, 40, 3), (-1, 4096, 0)])
def test_workspace_size_explicit_partitions(pt, maxlen, parts):
    B, Hq, Hkv, d = 8, 64, 8, 128
    size = pa.pa_decode_workspace_size(B, Hq, Hkv, d, 16, maxlen, pt)
    if parts == 0:
        assert size == 0
        assert pa.pa_decode_partition_tokens(B, Hq, Hkv, d, 16, maxlen, pt) == -1
    else:
        # partial outputs, 256-byte aligned, then the (max, sum) pairs
        rows = B * Hq * parts
        o_bytes = -(-rows * d * 4 // 256) * 256
        assert size == o_bytes + rows * 8
        assert pa.pa_decode_partition_tokens(B, Hq, Hkv, d, 16, maxlen, pt) == pt


@pytest.mark.parametrize("pt,maxlen,parts", [(512, 32768, 64), (-1, 4096, 1), (0, 2500, 1), (16, 40, 3)])
def test_shared_prefix_workspace_size(pt, maxlen, parts):
    """Two slots per partition (the shared items', then the sequence's own); a call that would
    not split still has one of each."""
    B, n, Hq, Hkv, d = 128, 4, 40, 40, 128
    size = pa.pa_decode_shared_prefix_workspace_size(B, n, Hq, Hkv, d, 16, maxlen, pt)
    rows = B * Hq * 2 * parts
    assert size == -(-rows * d * 4 // 256) * 256 + rows * 8
    assert pa.pa_decode_shared_prefix_workspace_size(0, n, Hq, Hkv, d, 16, maxlen, pt) == 0


def test_step_staging_size_shared_prefix():
    """The shared-prefix host step stages the plain step's sections plus one prefix length per group
    (256-byte aligned) and the shared-prefix decode's workspace in place of the plain one's."""
    B, n, mb, pairs, Hq, Hkv, d, bs, L = 128, 4, 160, 8, 40, 40, 128, 16, 2500
    plain = pa.pa_decode_step_staging_size(B, mb, pairs, Hq, Hkv, d, bs, L, 0)
    shared = pa.pa_decode_step_staging_size_shared_prefix(B, n, mb, pairs, Hq, Hkv, d, bs, L, 0)
    slack = 2 * 256 * 8  # a 256-byte aligned workspace slice per chunk
    ws_plain = pa.pa_decode_workspace_size(B, Hq, Hkv, d, bs, L, 0)
    ws_shared = pa.pa_decode_shared_prefix_workspace_size(B, n, Hq, Hkv, d, bs, L, 0)
    rnd = lambda x: -(-x // 256) * 256
    plain_ws = rnd(ws_plain + slack) if ws_plain else 0
    assert shared - plain == rnd(B // n * 4) + rnd(ws_shared + slack) - plain_ws
    for g in (0, 65):
        assert pa.pa_decode_step_staging_size_shared_prefix(B, g, mb, pairs, Hq, Hkv, d, bs, L, 0) == 0
    assert pa.pa_decode_step_staging_size_shared_prefix(0, n, mb, pairs, Hq, Hkv, d, bs, L, 0) == 0


def test_shared_prefix_argument_errors_need_no_gpu():
    f = lib.pa_decode_shared_prefix
    base = [_fake(), _fake(), None, None, _fake(), _fake(), _fake(), 4, _fake(), _fake(), 4, 8, 64, 8, 8, 128,
            16, 64, 0.1, -1, _fake(0x100000), 1 << 20, None, None]

    def call(**kw):
        a = list(base)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)

    assert call(a11=0) == pa.PA_OK                        # empty batch
    assert call(a9=None) == pa.PA_ERR_INVALID_ARG         # prefix_lens missing
    assert call(a10=0) == pa.PA_ERR_INVALID_ARG           # group size 0
    assert call(a10=65) == pa.PA_ERR_INVALID_ARG          # group size above 64
    assert call(a2=_fake()) == pa.PA_ERR_INVALID_ARG      # k_new without v_new
    assert call(a15=96) == pa.PA_ERR_UNSUPPORTED          # head_dim
    assert call(a20=None) == pa.PA_ERR_INVALID_ARG        # always merges: needs a workspace
    assert call(a21=16) == pa.PA_ERR_INVALID_ARG          # workspace too small


def test_host_step_argument_errors_need_no_gpu():
    f = lib.pa_decode_step_host
    base = [_fake(), _fake(), _fake(), _fake(), _fake(), 4, _fake(), None, 0, 0, _fake(), _fake(), 2, 64, 8, 2,
            128, 16, 64, 0.1, -1, 0, _fake(0x100000), 1 << 20, None, None]

    def call(**kw):
        a = list(base)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)

    assert call(a12=0) == pa.PA_OK                        # empty batch
    assert call(a21=-1) == pa.PA_ERR_INVALID_ARG          # num_chunks < 0
    assert call(a21=9) == pa.PA_ERR_INVALID_ARG           # more chunks than the library pipelines
    assert call(a16=96) == pa.PA_ERR_UNSUPPORTED          # head_dim
    assert call(a8=1) == pa.PA_ERR_INVALID_ARG            # pairs beyond max_copy_pairs
    assert call(a23=16) == pa.PA_ERR_INVALID_ARG          # staging too small
    assert call(a22=_fake(0x100010)) == pa.PA_ERR_INVALID_ARG  # staging not 256-byte aligned
    assert call(a20=24) == pa.PA_ERR_INVALID_ARG          # partition not a multiple of block_size


def test_fp8_host_step_rejects_bad_scales():
    """Scales that are not finite and positive are refused before anything is enqueued."""
    for ks, vs in ((0.0, 1.0), (1.0, -1.0), (float("inf"), 1.0), (1.0, float("nan"))):
        rc = lib.pa_decode_step_host_fp8(_fake(), _fake(), _fake(), _fake(), _fake(), 4, _fake(), None, 0, 0,
                                         _fake(), _fake(), 2, 64, 8, 2, 128, 16, 64, 0.1, ks, vs, -1, 0,
                                         _fake(0x100000), 1 << 20, None, None)
        assert rc == pa.PA_ERR_INVALID_ARG


def test_header_is_c99_and_links(tmp_path):
    """include/pa.h is a C header: a C99 program using it compiles, links against libpa.so and runs
    (the program only calls pa_version; its decode-step function shows one serving-loop step)."""
    import shutil
    import subprocess
    from paged_kv_cache_349_b200 import build as B
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "c_abi_example"
    lib_dir = os.path.dirname(B.LIB)
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "csrc", "c_abi_example.c"), "-L", lib_dir, "-lpa",
                           f"-Wl,-rpath,{lib_dir}", "-o", str(exe)])
    assert subprocess.run([str(exe)]).returncode == 0
