"""The C-ABI library without a GPU: it loads, exports every entry point
include/pa.h declares, sizes workspaces, and rejects bad arguments on the
host before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

from paged_kv_cache_391_b200 import build as pa_build
from paged_kv_cache_391_b200 import pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def L():
    pa_build.build()
    return pa.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(pa.EXPORTS)


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (pa_[a-z0-9_]+)$", out, flags=re.M))
    for name in _declared():
        assert name in exported, name
        assert hasattr(L, name)


def test_status_strings(L):
    assert pa.status_string(pa.PA_OK) == "ok"
    assert "workspace" in pa.status_string(pa.PA_ERR_WORKSPACE_TOO_SMALL)
    assert pa.last_cuda_error() == ""


def test_workspace_size(L):
    f = L.pa_decode_workspace_size
    assert f(8, 64, 128, 512, 512) == 0          # one partition: no split
    assert f(8, 64, 128, 131072, 0) == 0         # no split requested
    parts = 131072 // 512
    rows = 8 * 64 * parts
    want = -(-rows * 128 * 4 // 256) * 256 + -(-rows * 4 // 256) * 256
    assert f(8, 64, 128, 131072, 512) == want
    assert f(3, 4, 64, 513, 512) == (-(-3 * 4 * 2 * 64 * 4 // 256) * 256 + 256)


FAKE = 1 << 20  # a 16-byte aligned non-NULL address; never dereferenced


def _decode(L, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, stride=4, cl=FAKE, S=2, Hq=8, g=4, D=128,
             bs=16, NB=10, max_ctx=64, scale=0.1, P=512, ws=None, ws_bytes=0, err=None, dt=1)
    a.update(kw)
    return L.pa_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["stride"], a["cl"], a["S"],
                       a["Hq"], a["g"], a["D"], a["bs"], a["NB"], a["max_ctx"],
                       ctypes.c_float(a["scale"]), a["P"], a["ws"], a["ws_bytes"], a["err"],
                       a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(bs=8), pa.PA_ERR_UNSUPPORTED),
    (dict(D=96), pa.PA_ERR_UNSUPPORTED),
    (dict(g=3), pa.PA_ERR_UNSUPPORTED),
    (dict(g=32, Hq=32), pa.PA_ERR_UNSUPPORTED),
    (dict(P=500), pa.PA_ERR_UNSUPPORTED),
    (dict(out=None), pa.PA_ERR_INVALID_ARG),
    (dict(k=FAKE + 2), pa.PA_ERR_INVALID_ARG),
    (dict(stride=3), pa.PA_ERR_INVALID_ARG),
    (dict(dt=7), pa.PA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), pa.PA_ERR_INVALID_ARG),
    (dict(max_ctx=-1), pa.PA_ERR_INVALID_ARG),
    (dict(max_ctx=2048, stride=128), pa.PA_ERR_INVALID_ARG),        # needs a workspace
    (dict(max_ctx=2048, stride=128, ws=FAKE, ws_bytes=100), pa.PA_ERR_WORKSPACE_TOO_SMALL),
    (dict(S=0), pa.PA_OK),                                          # nothing to do
])
def test_decode_rejects_on_the_host(L, kw, status):
    assert _decode(L, **kw) == status


def test_write_kv_rejects_on_the_host(L):
    f = L.pa_write_kv
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 8, 10, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 100, 16, 10, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    assert f(None, FAKE, FAKE, FAKE, FAKE, 4, 8, 128, 16, 10, 1, None, None) == pa.PA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE + 8, FAKE, FAKE, 4, 8, 128, 16, 10, 1, None, None) == pa.PA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 8, 128, 16, 10, 1, None, None) == pa.PA_ERR_INVALID_ARG
    assert f(None, None, None, None, None, 0, 8, 128, 16, 10, 1, None, None) == pa.PA_OK


def test_copy_blocks_rejects_on_the_host(L):
    f = L.pa_copy_blocks
    arr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    bad = (ctypes.c_void_p * 2)(FAKE, None)
    P = ctypes.cast(arr, ctypes.c_void_p)
    assert f(P, P, 0, FAKE, 3, 8, 128, 16, 10, 1, None, None) == pa.PA_ERR_INVALID_ARG
    assert f(P, P, pa.PA_MAX_LAYERS + 1, FAKE, 3, 8, 128, 16, 10, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    assert f(P, P, 2, FAKE, 3, 8, 128, 8, 10, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    assert f(P, ctypes.cast(bad, ctypes.c_void_p), 2, FAKE, 3, 8, 128, 16, 10, 1, None, None) == \
        pa.PA_ERR_INVALID_ARG
    assert f(P, P, 2, FAKE, 0, 8, 128, 16, 10, 1, None, None) == pa.PA_OK


def test_missing_library_is_an_error(monkeypatch, tmp_path):
    monkeypatch.setattr(pa, "_lib", None)
    monkeypatch.setattr(pa, "LIB_PATH", str(tmp_path / "libpa.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        pa.lib()


def test_swap_blocks_rejects_on_the_host(L):
    f = L.pa_swap_blocks
    arr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    P = ctypes.cast(arr, ctypes.c_void_p)
    args = lambda **k: [k.get("sk", P), P, P, P, k.get("nl", 1), FAKE, k.get("n", 3), 8, 128,
                        k.get("bs", 16), 10, 10, k.get("dt", 1), None, None]
    assert f(*args(nl=0)) == pa.PA_ERR_INVALID_ARG
    assert f(*args(nl=pa.PA_MAX_LAYERS + 1)) == pa.PA_ERR_UNSUPPORTED
    assert f(*args(bs=8)) == pa.PA_ERR_UNSUPPORTED
    assert f(*args(dt=5)) == pa.PA_ERR_INVALID_ARG
    assert f(*args(sk=None)) == pa.PA_ERR_INVALID_ARG
    assert f(*args(n=0)) == pa.PA_OK
    # an address no allocation owns is refused before any launch
    assert f(*args()) == pa.PA_ERR_INVALID_ARG


def test_persistent_workspace_size(L):
    f, base = L.pa_decode_persistent_workspace_size, L.pa_decode_workspace_size
    assert f(0, 8, 128, 512, 512) == 0
    # one partition: no partials, but the work list (8 items) and the plan
    assert f(8, 64, 128, 512, 512) == 256 + 256
    parts = 131072 // 512
    assert f(8, 64, 128, 131072, 512) == (base(8, 64, 128, 131072, 512)
                                           + -(-8 * parts * 4 // 256) * 256 + 256)


def _decode_persistent(L, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, stride=4, cl=FAKE, S=2, Hq=8, g=4, D=128,
             bs=16, NB=10, max_ctx=64, scale=0.1, P=512, ws=None, ws_bytes=0, err=None, dt=1)
    a.update(kw)
    return L.pa_decode_persistent(a["out"], a["q"], a["k"], a["v"], a["bt"], a["stride"],
                                  a["cl"], a["S"], a["Hq"], a["g"], a["D"], a["bs"], a["NB"],
                                  a["max_ctx"], ctypes.c_float(a["scale"]), a["P"], a["ws"],
                                  a["ws_bytes"], a["err"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(), pa.PA_ERR_INVALID_ARG),                                 # always needs a workspace
    (dict(ws=FAKE + 16, ws_bytes=1 << 20), pa.PA_ERR_INVALID_ARG),   # not 256-byte aligned
    (dict(ws=FAKE, ws_bytes=511), pa.PA_ERR_WORKSPACE_TOO_SMALL),
    (dict(max_ctx=16 * 65537, stride=65537, P=16), pa.PA_ERR_UNSUPPORTED),  # > 65536 partitions
    (dict(g=3), pa.PA_ERR_UNSUPPORTED),
    (dict(S=0), pa.PA_OK),
])
def test_decode_persistent_rejects_on_the_host(L, kw, status):
    assert _decode_persistent(L, **kw) == status


def _decode_shared(L, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, stride=4, cl=FAKE, S=2, Hq=8, g=4, D=128,
             bs=16, NB=10, max_ctx=64, scale=0.1, shared=0, P=512, ws=None, ws_bytes=0, err=None,
             dt=1)
    a.update(kw)
    return L.pa_decode_shared_prefix(a["out"], a["q"], a["k"], a["v"], a["bt"], a["stride"],
                                     a["cl"], a["S"], a["Hq"], a["g"], a["D"], a["bs"], a["NB"],
                                     a["max_ctx"], ctypes.c_float(a["scale"]), a["shared"],
                                     a["P"], a["ws"], a["ws_bytes"], a["err"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(shared=-1), pa.PA_ERR_INVALID_ARG),
    (dict(shared=65), pa.PA_ERR_INVALID_ARG),                 # longer than max_context_len
    (dict(g=3), pa.PA_ERR_UNSUPPORTED),
    (dict(out=None, shared=32), pa.PA_ERR_INVALID_ARG),
    (dict(max_ctx=2048, stride=128, shared=1536), pa.PA_ERR_INVALID_ARG),  # needs a workspace
    (dict(max_ctx=2048, stride=128, shared=1536, ws=FAKE, ws_bytes=100),
     pa.PA_ERR_WORKSPACE_TOO_SMALL),
    (dict(S=0, shared=32), pa.PA_OK),                         # nothing to do
])
def test_decode_shared_prefix_rejects_on_the_host(L, kw, status):
    assert _decode_shared(L, **kw) == status


def _prefill(L, **kw):
    a = dict(out=FAKE, q=FAKE, qs=FAKE, nq=8, maxq=4, k=FAKE, v=FAKE, bt=FAKE, stride=4, cl=FAKE,
             S=2, Hq=8, g=4, D=128, bs=16, NB=10, max_ctx=64, scale=0.1, P=512, ws=None,
             ws_bytes=0, err=None, dt=1)
    a.update(kw)
    return L.pa_prefill_chunk(a["out"], a["q"], a["qs"], a["nq"], a["maxq"], a["k"], a["v"],
                              a["bt"], a["stride"], a["cl"], a["S"], a["Hq"], a["g"], a["D"],
                              a["bs"], a["NB"], a["max_ctx"], ctypes.c_float(a["scale"]), a["P"],
                              a["ws"], a["ws_bytes"], a["err"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(qs=None), pa.PA_ERR_INVALID_ARG),                  # q_start is required
    (dict(qs=FAKE + 2), pa.PA_ERR_INVALID_ARG),              # misaligned q_start
    (dict(maxq=-1), pa.PA_ERR_INVALID_ARG),
    (dict(nq=-1), pa.PA_ERR_INVALID_ARG),
    (dict(g=3), pa.PA_ERR_UNSUPPORTED),
    (dict(D=96), pa.PA_ERR_UNSUPPORTED),
    (dict(P=100), pa.PA_ERR_UNSUPPORTED),                    # not a multiple of 16
    (dict(max_ctx=2048, stride=128), pa.PA_ERR_INVALID_ARG),  # needs a workspace
    (dict(max_ctx=2048, stride=128, ws=FAKE, ws_bytes=100), pa.PA_ERR_WORKSPACE_TOO_SMALL),
    (dict(nq=0), pa.PA_OK),                                  # no query rows: nothing to do
    (dict(S=0), pa.PA_OK),
])
def test_prefill_chunk_rejects_on_the_host(L, kw, status):
    assert _prefill(L, **kw) == status


def test_read_probe_rejections(L):
    """pa_read_probe refuses bad methods, pointers, alignment and sizes on
    the host, before any launch."""
    f = L.pa_read_probe
    assert f(FAKE, 1 << 20, 3, FAKE, None, None) == pa.PA_ERR_INVALID_ARG      # method
    assert f(FAKE, 4096, 2, FAKE, None, None) == pa.PA_ERR_INVALID_ARG         # < two tiles
    assert f(None, 1 << 20, 0, FAKE, None, None) == pa.PA_ERR_INVALID_ARG      # buffer
    assert f(FAKE, 1 << 20, 0, None, None, None) == pa.PA_ERR_INVALID_ARG      # sink
    assert f(FAKE + 8, 1 << 20, 0, FAKE, None, None) == pa.PA_ERR_INVALID_ARG  # 16-byte base
    assert f(FAKE, (1 << 20) + 8, 1, FAKE, None, None) == pa.PA_ERR_INVALID_ARG  # 16-byte size
    assert f(FAKE, 0, 0, None, None, None) == pa.PA_OK                         # nothing to read


def test_chunk_workspace_size(L):
    """pa_prefill_chunk_workspace_size: the split partials of every query
    row, plus -- on the tcgen05 path only -- 8 bytes per possible (sequence,
    query-tile pair, partition) item and 256 bytes for the longest-first
    plan."""
    f, dws = L.pa_prefill_chunk_workspace_size, L.pa_decode_workspace_size
    r256 = lambda x: -(-x // 256) * 256  # noqa: E731
    # 16 sequences, 256-token chunks, group 4, D 128, no split: 1024 rows -> 8 tiles -> 4 pairs
    assert f(4096, 16, 32, 4, 128, 256, 8192, 0) == 0 + r256(16 * 4 * 1 * 8) + 256
    # split in 512-token partitions: 16 partitions of 8192 tokens
    parts = 8192 // 512
    assert f(4096, 16, 32, 4, 128, 256, 8192, 512) == \
        dws(4096, 32, 128, 8192, 512) + r256(16 * 4 * parts * 8) + 256
    # not the tcgen05 path: D 64, a partition size that is not a multiple of 128,
    # too few rows -- the partials only
    assert f(4096, 16, 32, 4, 64, 256, 8192, 512) == dws(4096, 32, 64, 8192, 512)
    assert f(4096, 16, 32, 4, 128, 256, 8192, 64) == dws(4096, 32, 128, 8192, 64)
    assert f(64, 16, 32, 4, 128, 4, 8192, 512) == dws(64, 32, 128, 8192, 512)
