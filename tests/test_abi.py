"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point that
include/gdn.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from linear_attention_10_b200 import build as gdn_build
from linear_attention_10_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def L():
    gdn_build.build()
    return gdn.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(gdn_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("gdn_chunk_prefill", "gdn_decode_step", "gdn_get_device_status", "gdn_status_string",
              "gdn_chunk_prefill_workspace_bytes", "gdn_version"):
        assert n in names
    assert set(names) == set(gdn.EXPORTS), names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    for code in range(0, -9, -1):
        s = gdn.status_string(code)
        assert s and "unknown" not in s
    assert "unknown" in gdn.status_string(-99)
    assert L.gdn_version() >= 100


def test_workspace_bytes(L):
    w = gdn.workspace_bytes
    assert w(4096, 1, 32, 128, 128) > 0
    assert w(0, 1, 32, 128, 128) > 0
    assert w(4096, 1, 32, 96, 128) == 0          # unsupported head size
    assert w(-1, 1, 32, 128, 128) == 0
    assert w(4096, 0, 32, 128, 128) == 0
    assert w(8192, 1, 32, 128, 128) >= w(4096, 1, 32, 128, 128)
    assert w(4096, 1, 32, 128, 128) % 256 == 0


def _restated_workspace(T, NS, H):
    """The prefill workspace as the header describes it: 256-byte aligned regions (meta int32[8],
    table offsets int32[NS+1], the table int4[T/32 + NS], segments int32[6 NS + 1], the scan order
    int32[NS]) and the operator records, [T/32 + NS][H] x 16,896 B (fp32 path) or [T/64 + NS][H] x
    49,664 B (bf16 path), whichever is larger."""
    al = lambda x: (x + 255) & ~255
    nc, npair = T // 32 + NS, T // 64 + NS
    regions = [8 * 4, (NS + 1) * 4, nc * 16, (6 * NS + 1) * 4, NS * 4, max(nc * H * 16896, npair * H * 49664)]
    return sum(al(r) for r in regions)


def test_workspace_bytes_match_the_documented_layout(L):
    for T, NS, H, dk, dv in [(4096, 1, 32, 128, 128), (24709, 4, 32, 128, 128), (100, 3, 4, 64, 64),
                             (0, 1, 2, 64, 128), (131072, 1, 32, 128, 128), (63, 7, 1, 128, 64)]:
        assert gdn.workspace_bytes(T, NS, H, dk, dv) == _restated_workspace(T, NS, H), (T, NS, H, dk, dv)


def test_scratch_limit_stated_in_the_header(L):
    """The allocation-free entry point's 64 MiB scratch holds one bf16 sequence of about 2,680 tokens at
    H = 32, d = 128 (include/gdn.h): the largest length whose workspace fits."""
    lo, hi = 1, 1 << 20
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if gdn.workspace_bytes(mid, 1, 32, 128, 128) <= 64 << 20:
            lo = mid
        else:
            hi = mid - 1
    assert 2600 <= lo <= 2700, lo


FAKE = 1 << 20   # 16-byte aligned non-null address; never dereferenced on these paths


def prefill(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu=FAKE, N=1, T=64, s_in=None, out=FAKE,
             s_out=FAKE, H=2, dk=64, dv=64, dtype=1, ws=FAKE, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return L.gdn_chunk_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["cu"], a["N"], a["T"], a["s_in"],
                               a["out"], a["s_out"], a["H"], a["dk"], a["dv"], a["dtype"], a["ws"],
                               a["ws_bytes"], a["stream"])


def test_prefill_rejects_bad_arguments(L):
    assert prefill(L, q=None) == -1
    assert prefill(L, out=None) == -1
    assert prefill(L, N=0) == -1
    assert prefill(L, H=0) == -1
    assert prefill(L, T=-1) == -1
    assert prefill(L, dtype=7) == -1
    assert prefill(L, cu=None, N=3, T=64) == -1        # 64 tokens do not split into 3 equal sequences
    assert prefill(L, dk=96) == -2
    assert prefill(L, dv=32) == -2
    assert prefill(L, k=FAKE + 4) == -3
    assert prefill(L, s_out=FAKE + 8) == -3
    assert prefill(L, beta=FAKE + 2) == -3
    assert prefill(L, cu=FAKE + 1) == -3
    assert prefill(L, ws=None) == -5
    assert prefill(L, ws=FAKE + 16) == -5              # workspace must be 256-byte aligned
    assert prefill(L, ws_bytes=16) == -5


def decode(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, s=FAKE, out=FAKE, B=4, H=2, dk=128, dv=128, dtype=1,
             stream=None)
    a.update(kw)
    return L.gdn_decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["s"], a["out"], a["B"], a["H"],
                             a["dk"], a["dv"], a["dtype"], a["stream"])


def test_decode_rejects_bad_arguments(L):
    assert decode(L, s=None) == -1
    assert decode(L, H=0) == -1
    assert decode(L, B=-1) == -1
    assert decode(L, dtype=3) == -1
    assert decode(L, dk=32) == -2
    assert decode(L, v=FAKE + 2) == -3
    assert decode(L, g=FAKE + 2) == -3
    assert decode(L, B=0) == 0                          # nothing to do, nothing enqueued


def verify(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, s=FAKE, st=FAKE, out=FAKE, B=4, Tk=3, H=2, dk=128, dv=128,
             dtype=1, stream=None)
    a.update(kw)
    return L.gdn_decode_verify(a["q"], a["k"], a["v"], a["g"], a["beta"], a["s"], a["st"], a["out"], a["B"],
                               a["Tk"], a["H"], a["dk"], a["dv"], a["dtype"], a["stream"])


def test_verify_rejects_bad_arguments(L):
    assert verify(L, s=None) == -1
    assert verify(L, st=None, out=None) == -1           # nothing to return
    assert verify(L, Tk=0) == -1
    assert verify(L, H=0) == -1
    assert verify(L, B=-1) == -1
    assert verify(L, dtype=3) == -1
    assert verify(L, dv=96) == -2
    assert verify(L, st=FAKE + 4) == -3
    assert verify(L, beta=FAKE + 1) == -3
    assert verify(L, B=0) == 0                          # nothing to do, nothing enqueued


def verify_tree(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, par=FAKE, s=FAKE, st=FAKE, out=FAKE, B=4, Tk=3, H=2,
             dk=128, dv=128, dtype=1, stream=None)
    a.update(kw)
    return L.gdn_decode_verify_tree(a["q"], a["k"], a["v"], a["g"], a["beta"], a["par"], a["s"], a["st"], a["out"],
                                    a["B"], a["Tk"], a["H"], a["dk"], a["dv"], a["dtype"], a["stream"])


def test_verify_tree_rejects_bad_arguments(L):
    """Every case returns before any launch (the pointers are not real device memory)."""
    assert verify_tree(L, par=None) == -1
    assert verify_tree(L, st=None) == -1                # the tree reads parents' states back from it
    assert verify_tree(L, s=None) == -1
    assert verify_tree(L, Tk=0) == -1
    assert verify_tree(L, dtype=3) == -1
    assert verify_tree(L, dv=96) == -2
    assert verify_tree(L, par=FAKE + 2) == -3
    assert verify_tree(L, st=FAKE + 4) == -3
    assert verify_tree(L, B=0) == 0                     # nothing to do, nothing enqueued


def test_status_string_names_bad_parents(L):
    assert b"BAD_PARENTS" in L.gdn_status_string(-9)


def test_selftest_rejects_out_of_range_limits(L):
    """Both limits are refused before any launch."""
    assert L.gdn_selftest_wait_timeout(999_999, None) == -1
    assert L.gdn_selftest_wait_timeout(2_000_000_001, None) == -1


def prefill_cuts(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu=FAKE, N=2, T=64, cuts=FAKE, nc=2, s_in=None, out=FAKE,
             s_out=FAKE, snaps=FAKE, H=2, dk=128, dv=128, dtype=1, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.gdn_chunk_prefill_cuts(a["q"], a["k"], a["v"], a["g"], a["beta"], a["cu"], a["N"], a["T"], a["cuts"],
                                    a["nc"], a["s_in"], a["out"], a["s_out"], a["snaps"], a["H"], a["dk"], a["dv"],
                                    a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


def test_prefill_cuts_rejects_bad_arguments(L):
    assert prefill_cuts(L, nc=0) == -1
    assert prefill_cuts(L, cuts=None) == -1
    assert prefill_cuts(L, snaps=None) == -1
    assert prefill_cuts(L, snaps=FAKE + 8) == -3
    assert prefill_cuts(L, cuts=FAKE + 2) == -3
    assert prefill_cuts(L, dk=96) == -2
    # the workspace must cover num_seqs + num_cuts segments
    need_plain = L.gdn_chunk_prefill_workspace_bytes(64, 2, 2, 128, 128)
    need_cuts = L.gdn_chunk_prefill_workspace_bytes(64, 2 + 2, 2, 128, 128)
    assert need_cuts > need_plain
    assert prefill_cuts(L, ws_bytes=need_cuts - 1) == -5


def test_normalisation_flag(L):
    assert L.gdn_chunk_prefill_workspace_bytes_ex(4096, 1, 32, 128, 128, 1) == \
        L.gdn_chunk_prefill_workspace_bytes(4096, 1, 32, 128, 128)
    plain = L.gdn_chunk_prefill_workspace_bytes(4096, 1, 32, 128, 128)
    assert L.gdn_chunk_prefill_workspace_bytes_ex(4096, 1, 32, 128, 128, 1 | gdn.GDN_QK_L2NORM) >= plain + 2 * 4096 * 32 * 128 * 2
    assert L.gdn_chunk_prefill_workspace_bytes_ex(4096, 1, 32, 128, 128, 0x200) == 0      # unknown flag bit
    assert prefill(L, dtype=1 | 0x200) == -1
    assert decode(L, dtype=1 | 0x200) == -1
    assert verify(L, dtype=1 | 0x200) == -1
    # the normalised copies need room: the plain workspace size of the same call is refused (the
    # sizes here are prefill()'s defaults: T=64, N=1, H=2, dk=dv=64)
    need = L.gdn_chunk_prefill_workspace_bytes(64, 1, 2, 64, 64)
    need_ex = L.gdn_chunk_prefill_workspace_bytes_ex(64, 1, 2, 64, 64, 1 | gdn.GDN_QK_L2NORM)
    assert need_ex > need
    assert prefill(L, dtype=1 | gdn.GDN_QK_L2NORM, ws_bytes=need) == -5
    assert prefill(L, dtype=1 | gdn.GDN_QK_L2NORM, ws_bytes=need_ex - 1) == -5


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(gdn, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(gdn, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        gdn.lib()
