"""The C-ABI boundary on a machine without a GPU: liblsa.so loads, exports every entry point
that include/lsa.h declares, and rejects bad arguments on the host before any device work."""
import ctypes
import os
import re

import pytest

from lightning_indexer_top_score_b200 import build as lsa_build
from lightning_indexer_top_score_b200 import lsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "lsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    lsa_build.build()
    return lsa.load()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert set(names) == set(lsa.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n
    out = os.popen(f"nm -D --defined-only {lsa.LIB_PATH}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", out), n


def test_status_strings_and_version(lib):
    for code, name in lsa.STATUS.items():
        assert lib.lsa_status_string(code).decode() == name
    assert lib.lsa_version() >= 100


def test_workspace_queries(lib):
    n = lsa.lsa_index_workspace_bytes(32, 1, 64, 128, 131072, 1008)
    # flat scores (4 B/token) + candidate slots (4 B/token) dominate
    assert n >= 32 * 131072 * 8
    assert lsa.lsa_index_workspace_bytes(4, 1, 64, 128, 1 << 20, 1008, 128, 8, 1024) > 0
    assert lsa.lsa_index_workspace_bytes(1, 1, 64, 96, 1000, 10) == 0      # D_I unsupported
    assert lsa.lsa_index_workspace_bytes(1, 1, 64, 128, 1000, 5000) == 0   # K > 4096
    assert lsa.lsa_index_workspace_bytes(1, 1, 64, 128, 1000, 10, 100, 8, 4) == 0  # page
    assert lsa.lsa_attend_workspace_bytes(32, 1, 128, 512, 1008, 16, 1024) >= 256
    assert lsa.lsa_attend_workspace_bytes(1, 1, 12, 512, 10, 0, 0) == 0    # H % 8


def test_host_validation_before_device_work(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)  # never dereferenced: validation fails first
    # null pointers
    st = lib.lsa_index(None, fake, fake, None, fake, fake, 1, 1, 64, 128, 1024, 16, 16, 64, 128,
                       8, 0, fake, None, None, fake, 1 << 30, None)
    assert st == 1
    # HI requested without a mean cache
    st = lib.lsa_index(fake, fake, fake, None, fake, fake, 1, 1, 64, 128, 1024, 16, 16, 64, 128,
                       8, 4, fake, None, None, fake, 1 << 30, None)
    assert st == 1
    # unsupported head dim
    st = lib.lsa_index(fake, fake, fake, None, fake, fake, 1, 1, 64, 96, 1024, 16, 16, 64, 128,
                       8, 0, fake, None, None, fake, 1 << 30, None)
    assert st == 2
    # short workspace
    st = lib.lsa_index(fake, fake, fake, None, fake, fake, 1, 1, 64, 128, 1024, 16, 16, 64, 128,
                       8, 0, fake, None, None, fake, 64, None)
    assert st == 3
    # attention: unsupported latent width, NaN scale, short workspace
    st = lib.lsa_attend(fake, fake, fake, fake, fake, 1, 1, 128, 512, 512, 1024, 16, 16, 64,
                        ctypes.c_float(0.04), fake, fake, fake, 1 << 30, None)
    assert st == 2
    st = lib.lsa_attend(fake, fake, fake, fake, fake, 1, 1, 128, 576, 512, 1024, 16, 16, 64,
                        ctypes.c_float(float("nan")), fake, fake, fake, 1 << 30, None)
    assert st == 1
    for bad in (-0.04, 0.0, float("inf")):  # the softmax scale must be positive and finite
        st = lib.lsa_attend(fake, fake, fake, fake, fake, 1, 1, 128, 576, 512, 1024, 16, 16, 64,
                            ctypes.c_float(bad), fake, fake, fake, 1 << 30, None)
        assert st == 1
    st = lib.lsa_attend(fake, fake, fake, fake, fake, 1, 1, 128, 576, 512, 1024, 16, 16, 64,
                        ctypes.c_float(0.04), fake, fake, fake, 8, None)
    assert st == 3
    # append: nothing to append / missing destination
    st = lib.lsa_kv_append(None, None, None, None, None, fake, 1, 1, 128, 576, 1024, 8, None, None)
    assert st == 1
    st = lib.lsa_kv_append(fake, None, None, None, None, fake, 1, 1, 128, 576, 1024, 8, None, None)
    assert st == 1
    st = lib.lsa_get_error(None, None, None)
    assert st == 1
    # backward: (q, c, idx, kv_len, q_pos, B, T, H, D_qk, D_v, L_max, K, sink, swa, scale,
    #            out, lse, dout, dq, dc, err, stream)
    f = ctypes.c_float(0.04)

    def bwd(**kw):
        a = dict(q=fake, idx=fake, H=128, D_qk=576, scale=f, out=None, lse=None, dq=fake, dc=fake)
        a.update(kw)
        return lib.lsa_attend_bwd(a["q"], fake, a["idx"], fake, fake, 1, 1, a["H"], a["D_qk"], 512,
                                  1024, 16, 16, 64, a["scale"], a["out"], a["lse"], fake, a["dq"],
                                  a["dc"], None, None)
    assert bwd(dq=None) == 1                       # missing output
    assert bwd(idx=None) == 1                      # K_sparse > 0 without indices
    assert bwd(out=fake) == 1                      # out without lse
    assert bwd(H=48) == 2                          # heads come in groups of 32
    assert bwd(D_qk=512) == 2                      # latent rows are 576 wide
    assert bwd(scale=ctypes.c_float(float("nan"))) == 1
    assert bwd(dc=P(0x1008)) == 1                  # vector atomics need 16-byte rows
    # FP8 quantiser and indexer: missing pointers, unsupported head dim
    assert lib.lsa_quantize_fp8(None, 128, 4, 128, fake, 128, fake, 1, None, None) == 1
    st = lib.lsa_index_fp8(fake, fake, fake, fake, fake, fake, fake, 1, 1, 64, 96, 1024, 16, 16, 64,
                           fake, None, fake, 1 << 30, None)
    assert st == 2


def test_minmax_entry_points_validate_on_the_host(lib):
    """MinMax pooling (Table 11): the cache refresh and the indexer refuse bad arguments before
    any device work."""
    P = ctypes.c_void_p
    ok, off = P(0x1000), P(0x1002)

    def kv(k=ok, kmm=ok, kv_old=ok, B=1, n_new=1, D=128, L=1024, sub=8):
        return lib.lsa_kv_minmax(k, kmm, kv_old, B, n_new, D, L, sub, None, None)
    assert kv(k=None) == 1
    assert kv(kmm=None) == 1
    assert kv(kv_old=None) == 1
    assert kv(n_new=-1) == 1
    assert kv(sub=0) == 1
    assert kv(D=96) == 2
    assert kv(k=off) == 1
    assert kv(kmm=off) == 1
    assert kv(n_new=0) == 0     # nothing to append: no launch

    def index(kmm=ok, M=4, D=128):
        return lib.lsa_index_minmax(ok, ok, ok, kmm, ok, ok, 1, 1, 64, D, 1024, 16, 16, 64, 128,
                                    8, M, ok, None, None, ok, 1 << 30, None)
    assert index(M=0) == 1      # MinMax pooling is a stage-1 variant: M >= 1
    assert index(kmm=None) == 1
    assert index(D=96) == 2


def test_misaligned_pointers_are_refused_on_the_host(lib):
    """bf16 rows are read with 16-byte vector loads, cp.async and TMA: a pointer off a 16-byte
    boundary (a contiguous bf16 tensor at an odd element offset) is refused before any launch
    instead of faulting on the device."""
    P = ctypes.c_void_p
    ok, off = P(0x1000), P(0x1002)
    f = ctypes.c_float(0.04)

    def index(q=ok, w=ok, k=ok, km=None, M=0, ws=ok):
        return lib.lsa_index(q, w, k, km, ok, ok, 1, 1, 64, 128, 1024, 16, 16, 64, 128, 8, M,
                             ok, None, None, ws, 1 << 30, None)
    assert index(q=off) == 1
    assert index(k=off) == 1
    assert index(km=off, M=4) == 1
    assert index(ws=off) == 1
    assert index(w=P(0x1001)) == 1

    def attend(q=ok, c=ok, out=ok, lse=ok):
        return lib.lsa_attend(q, c, ok, ok, ok, 1, 1, 128, 576, 512, 1024, 16, 16, 64, f, out, lse,
                              ok, 1 << 30, None)
    assert attend(q=off) == 1
    assert attend(c=off) == 1
    assert attend(out=off) == 1
    assert attend(lse=off) == 1

    def append(kn=ok, k=ok, km=None, cn=None, c=None):
        return lib.lsa_kv_append(kn, k, km, cn, c, ok, 1, 1, 128, 576, 1024, 8, None, None)
    assert append(kn=off) == 1
    assert append(k=off) == 1
    assert append(km=off) == 1
    assert append(kn=None, k=None, cn=off, c=ok) == 1
    assert append(kn=None, k=None, cn=ok, c=off) == 1
    st = lib.lsa_index_fp8(off, ok, ok, ok, ok, ok, ok, 1, 1, 64, 128, 1024, 16, 16, 64, ok, None,
                           ok, 1 << 30, None)
    assert st == 1
    st = lib.lsa_index_noalloc(off, ok, ok, None, ok, ok, 1, 1, 64, 128, 1024, 16, 16, 64, 128, 8,
                               0, ok, None, None)
    assert st in (1, 4)  # refused on the host (4 if the scratch lookup already needs a device)


def test_binding_refuses_cpu_tensors(lib):
    torch = pytest.importorskip("torch")
    x = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lsa.lsa_index(x, x[..., 0], x[0], None, torch.zeros(1, dtype=torch.int32),
                      torch.zeros(1, 1, dtype=torch.int32), 16, 16, 64,
                      ws=torch.zeros(1 << 20, dtype=torch.uint8))
