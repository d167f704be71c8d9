"""The C-ABI library on the host (no GPU work): it loads, exports every entry
point include/ssm_scan.h declares, and rejects bad arguments before anything
is enqueued. Every call here with fake pointers is one the library must
reject on the host; none of them can reach a kernel launch."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_scan.h")

from selective_state_space_39_b200 import _binding as bnd  # noqa: E402


@pytest.fixture(scope="module")
def L():
    from selective_state_space_39_b200 import build
    build.build()
    return bnd.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssm_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ["ssm_scan_fwd", "ssm_state_update", "ssm_scan_workspace_bytes",
                 "ssm_scan_plan", "ssm_scan_status", "ssm_status_string", "ssm_scan_version"]:
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), f"libssmscan.so does not export {name}"


def test_version_and_status_strings(L):
    assert L.ssm_scan_version() >= 10000
    assert L.ssm_status_string(0) == b"ok"
    assert L.ssm_status_string(-1) == b"invalid argument"
    assert L.ssm_status_string(-5) == b"a kernel wait timed out"
    assert L.ssm_status_string(12345) == b"unknown status"


def test_plan_splits_long_sequences(L):
    p = bnd.ScanPlan()
    assert L.ssm_scan_plan(1, 262144, 1536, 16, 1, ctypes.byref(p)) == 0
    assert p.segments > 1 and p.segment_steps % 16 == 0
    assert (p.segments - 1) * p.segment_steps < 262144 <= p.segments * p.segment_steps
    assert p.kernels == (3 if p.segments > 9 else 2)
    assert p.channels_per_cta == 256 and p.channel_tiles == 6
    assert p.ctas_main == p.segments * 6 and p.ctas_carry == (p.segments - 1) * 6
    assert p.workspace_bytes == L.ssm_scan_workspace_bytes(1, 262144, 1536, 16, 1)
    q = bnd.ScanPlan()
    assert L.ssm_scan_plan(1, 1, 64, 16, 0, ctypes.byref(q)) == 0
    assert q.segments == 1 and q.kernels == 1


def test_plan_respects_forced_segments(L, monkeypatch):
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", "3")
    p = bnd.ScanPlan()
    assert L.ssm_scan_plan(2, 100, 64, 16, 0, ctypes.byref(p)) == 0
    assert p.segments == 3 and p.segment_steps == 48
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", "1000")
    assert L.ssm_scan_plan(2, 100, 64, 16, 0, ctypes.byref(p)) == 0
    assert p.segments == 7 and p.segment_steps == 16  # at most one segment per 16-step tile


def test_unsupported_sizes(L):
    p = bnd.ScanPlan()
    assert L.ssm_scan_plan(1, 8, 8, 3, 0, ctypes.byref(p)) == -2   # odd dstate
    assert L.ssm_scan_plan(1, 8, 8, 128, 0, ctypes.byref(p)) == -2  # above 64
    assert L.ssm_scan_plan(1, 8, 8, 16, 7, ctypes.byref(p)) == -2   # io dtype
    assert L.ssm_scan_plan(-1, 8, 8, 16, 0, ctypes.byref(p)) == -1
    assert L.ssm_scan_plan(1, 8, 8, 0, 0, ctypes.byref(p)) == -1
    assert L.ssm_scan_workspace_bytes(1, 8, 8, 3, 0) == 0


FAKE = 1 << 20  # an aligned address that is never dereferenced: every call below is rejected first
# Fake-pointer calls run only on machines without a GPU, so that a regression
# in host-side validation can never turn one into a kernel launch.
no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="fake-pointer validation tests run only without a GPU")


def scan(L, **kw):
    a = dict(batch=2, seqlen=32, dim=64, dstate=16, io=1, x=FAKE, delta=FAKE + 4096,
             A=FAKE + 8192, B=FAKE + 12288, C=FAKE + 16384, D=None, z=None, bias=None, sp=1,
             h0=None, y=FAKE + 65536 * 4, h_last=None, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return L.ssm_scan_fwd(a["batch"], a["seqlen"], a["dim"], a["dstate"], a["io"], a["x"],
                          a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"], a["sp"],
                          a["h0"], a["y"], a["h_last"], a["ws"], a["ws_bytes"], a["stream"])


@no_gpu_only
def test_scan_rejects_bad_arguments(L):
    assert scan(L, x=None) == -1
    assert scan(L, A=None) == -1
    assert scan(L, y=None) == -1
    assert scan(L, x=FAKE + 1) == -1            # misaligned bf16
    assert scan(L, io=0, B=FAKE + 12290) == -1  # misaligned fp32
    assert scan(L, h0=FAKE + 4) == -1           # h0 needs 8-byte alignment
    assert scan(L, A=FAKE + 8192 + 4) == -1     # rows of A are read as pairs
    assert scan(L, y=FAKE + 2) == -1            # y overlaps x
    assert scan(L, dstate=5) == -2
    assert scan(L, seqlen=-3) == -1
    assert scan(L) == -3                        # no workspace
    need = L.ssm_scan_workspace_bytes(2, 32, 64, 16, 1)
    assert scan(L, ws=FAKE * 64, ws_bytes=need - 1) == -3
    assert scan(L, ws=FAKE * 64 + 8, ws_bytes=need) == -3  # workspace not 16-byte aligned
    assert scan(L, batch=0) == 0 and scan(L, dim=0) == 0   # empty problems do nothing


@no_gpu_only
def test_state_update_rejects_bad_arguments(L):
    def upd(**kw):
        a = dict(batch=4, dim=64, dstate=16, io=1, state=FAKE, x=FAKE + 65536, delta=FAKE + 69632,
                 A=FAKE + 73728, B=FAKE + 81920, C=FAKE + 86016, D=None, z=None, bias=None, sp=1,
                 y=FAKE + 131072, stream=None)
        a.update(kw)
        return L.ssm_state_update(a["batch"], a["dim"], a["dstate"], a["io"], a["state"], a["x"],
                                  a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                                  a["sp"], a["y"], a["stream"])
    assert upd(state=None) == -1
    assert upd(state=FAKE + 8) == -1   # state needs 16-byte alignment for dstate % 4 == 0
    assert upd(A=FAKE + 73728 + 8) == -1  # A rows are read as 16-byte vectors
    assert upd(B=FAKE + 81922) == -1   # B is read four bf16 elements at a time
    assert upd(y=FAKE + 65536) == -1   # y overlaps x
    assert upd(y=FAKE + 64) == -1      # y overlaps the state
    assert upd(dstate=7) == -2
    assert upd(C=None) == -1
    assert upd(batch=0) == 0


@no_gpu_only
def test_scan_bwd_rejects_bad_arguments(L):
    K = 1 << 16  # spacing of the fake buffers: none of them overlap

    def bwd(**kw):
        a = dict(batch=2, seqlen=32, dim=64, dstate=16, io=1, x=FAKE, delta=FAKE + K,
                 A=FAKE + 2 * K, B=FAKE + 3 * K, C=FAKE + 4 * K, D=None, z=FAKE + 5 * K,
                 bias=None, sp=1, h0=None, dy=FAKE + 6 * K, dh_last=None, dx=FAKE + 7 * K,
                 ddelta=FAKE + 8 * K, dA=FAKE + 9 * K, dB=FAKE + 10 * K, dC=FAKE + 11 * K,
                 dD=None, dz=FAKE + 12 * K, dbias=None, dh0=None, ws=None, ws_bytes=0)
        a.update(kw)
        return L.ssm_scan_bwd(a["batch"], a["seqlen"], a["dim"], a["dstate"], a["io"], a["x"],
                              a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                              a["sp"], a["h0"], a["dy"], a["dh_last"], a["dx"], a["ddelta"],
                              a["dA"], a["dB"], a["dC"], a["dD"], a["dz"], a["dbias"], a["dh0"],
                              a["ws"], a["ws_bytes"], None)
    assert bwd(dz=None) == -1                 # z given without dz
    assert bwd(z=None) == -1                  # dz given without z
    assert bwd(dy=None) == -1
    assert bwd(dA=None) == -1
    assert bwd(dx=FAKE + 1) == -1             # misaligned bf16
    assert bwd(dB=FAKE + 10 * K + 2) == -1    # misaligned fp32
    assert bwd(dx=FAKE + 6 * K + 64) == -1    # dx overlaps dy
    assert bwd(dC=FAKE + 10 * K + 64) == -1   # dC overlaps dB
    assert bwd(dstate=32) == -2               # the backward supports dstate <= 16
    assert bwd(io=3) == -2
    assert bwd() == -3                        # no workspace
    need = L.ssm_scan_bwd_workspace_bytes(2, 32, 64, 16, 1)
    assert need > 0 and L.ssm_scan_bwd_workspace_bytes(2, 32, 64, 32, 1) == 0
    assert bwd(ws=FAKE * 64, ws_bytes=need - 1) == -3
    assert bwd(batch=0) == 0 and bwd(dim=0) == 0


@no_gpu_only
def test_conv_rejects_bad_arguments(L):
    K = 1 << 16

    def fwd(**kw):
        a = dict(batch=2, seqlen=32, dim=64, width=4, io=1, x=FAKE, w=FAKE + K, bias=None, silu=1,
                 out=FAKE + 2 * K)
        a.update(kw)
        return L.ssm_conv1d_silu_fwd(a["batch"], a["seqlen"], a["dim"], a["width"], a["io"],
                                     a["x"], a["w"], a["bias"], a["silu"], a["out"], None)

    def bwd(**kw):
        a = dict(batch=2, seqlen=32, dim=64, width=4, io=1, x=FAKE, w=FAKE + K, bias=None, silu=1,
                 dout=FAKE + 2 * K, dx=FAKE + 3 * K, dw=FAKE + 4 * K, db=FAKE + 5 * K, ws=None,
                 ws_bytes=0)
        a.update(kw)
        return L.ssm_conv1d_silu_bwd(a["batch"], a["seqlen"], a["dim"], a["width"], a["io"],
                                     a["x"], a["w"], a["bias"], a["silu"], a["dout"], a["dx"],
                                     a["dw"], a["db"], a["ws"], a["ws_bytes"], None)
    assert fwd(x=None) == -1 and fwd(w=None) == -1 and fwd(out=None) == -1
    assert fwd(width=5) == -2 and fwd(width=1) == -2 and fwd(io=2) == -2
    assert fwd(out=FAKE + 64) == -1     # out overlaps x
    assert fwd(out=FAKE + 2 * K + 1) == -1  # misaligned bf16
    assert fwd(seqlen=0) == 0 and fwd(batch=0) == 0
    assert bwd(dx=FAKE + 2 * K + 64) == -1  # dx overlaps dout
    assert bwd(dw=FAKE + K) == -1       # dw overlaps w
    assert bwd(dout=None) == -1
    assert bwd() == -3                  # no workspace
    need = L.ssm_conv1d_silu_bwd_workspace_bytes(2, 32, 64, 4, 1)
    assert need > 0 and bwd(ws=FAKE * 64, ws_bytes=need - 1) == -3
    # decode step: state (2, 64, 3) bf16 = 768 bytes
    upd = lambda **kw: L.ssm_conv1d_silu_update(  # noqa: E731
        kw.get("batch", 2), 64, kw.get("width", 4), 1, kw.get("state", FAKE), kw.get("x", FAKE + K),
        FAKE + 2 * K, None, 1, kw.get("out", FAKE + 3 * K), None)
    assert upd(state=None) == -1 and upd(x=None) == -1
    assert upd(out=FAKE + 64) == -1     # out overlaps the state
    assert upd(width=6) == -2 and upd(batch=0) == 0


@no_gpu_only
def test_sequence_split_helpers_reject_bad_arguments(L):
    K = 1 << 16
    assert L.ssm_delta_sum(2, 32, 64, 1, None, None, 1, FAKE, None) == -1  # delta missing
    assert L.ssm_delta_sum(2, 32, 64, 1, FAKE, None, 1, FAKE + 64, None) == -1  # overlap
    assert L.ssm_delta_sum(2, 32, 64, 7, FAKE, None, 1, FAKE + K, None) == -2
    assert L.ssm_delta_sum(0, 32, 64, 1, FAKE, None, 1, FAKE + K, None) == 0
    assert L.ssm_compose_carries(2, 2, 64, 16, FAKE, None, None, None, FAKE + K, None) == -1
    assert L.ssm_compose_carries(-1, 2, 64, 16, FAKE, None, FAKE + 2 * K, FAKE + 3 * K,
                                 FAKE + K, None) == -1
    assert L.ssm_compose_carries(1, 2, 64, 16, FAKE, None, FAKE + 2 * K, FAKE + 3 * K,
                                 FAKE + 2 * K + 64, None) == -1  # h_in overlaps hend_all
    assert L.ssm_compose_carries(1, 0, 64, 16, FAKE, None, FAKE + 2 * K, FAKE + 3 * K,
                                 FAKE + K, None) == 0


@no_gpu_only
def test_ssd_rejects_bad_arguments(L):
    K = 1 << 18  # spacing of the fake buffers: none of them overlap

    def ssd(**kw):
        a = dict(batch=2, seqlen=64, nheads=2, headdim=64, dstate=128, io=1, x=FAKE, dt=FAKE + K,
                 A=FAKE + 2 * K, B=FAKE + 3 * K, C=FAKE + 4 * K, D=None, bias=None, sp=1, h0=None,
                 y=FAKE + 5 * K, h_last=None)
        a.update(kw)
        return L.ssm_ssd_scan_fwd(a["batch"], a["seqlen"], a["nheads"], a["headdim"],
                                  a["dstate"], a["io"], a["x"], a["dt"], a["A"], a["B"], a["C"],
                                  a["D"], a["bias"], a["sp"], a["h0"], a["y"], a["h_last"], None)
    assert ssd(io=0) == -2            # fp32 io: the tensor-core path is bf16
    assert ssd(io=7) == -1
    assert ssd(headdim=32) == -2
    assert ssd(dstate=16) == -2
    assert ssd(dstate=0) == -1
    assert ssd(batch=-1) == -1
    assert ssd(x=None) == -1
    assert ssd(A=None) == -1
    assert ssd(y=None) == -1
    assert ssd(x=FAKE + 8) == -1       # x needs 16-byte alignment
    assert ssd(B=FAKE + 3 * K + 2) == -1
    assert ssd(h0=FAKE + 6 * K + 4) == -1  # h0 needs 8-byte alignment
    assert ssd(y=FAKE + 16) == -1      # y overlaps x
    assert ssd(h_last=FAKE + 3 * K) == -1  # h_last overlaps B
    assert ssd(batch=0) == 0
    assert ssd(nheads=0) == 0


@no_gpu_only
def test_ssd_state_update_rejects_bad_arguments(L):
    K = 1 << 20

    def upd(**kw):
        a = dict(batch=2, nheads=4, headdim=64, dstate=128, io=1, state=FAKE, x=FAKE + K,
                 dt=FAKE + 2 * K, A=FAKE + 3 * K, B=FAKE + 4 * K, C=FAKE + 5 * K, D=None,
                 bias=None, sp=1, y=FAKE + 6 * K)
        a.update(kw)
        return L.ssm_ssd_state_update(a["batch"], a["nheads"], a["headdim"], a["dstate"],
                                      a["io"], a["state"], a["x"], a["dt"], a["A"], a["B"],
                                      a["C"], a["D"], a["bias"], a["sp"], a["y"], None)
    assert upd(dstate=16) == -2
    assert upd(dstate=0) == -1
    assert upd(io=5) == -1
    assert upd(batch=-1) == -1
    assert upd(state=None) == -1
    assert upd(A=None) == -1
    assert upd(y=None) == -1
    assert upd(state=FAKE + 8) == -1         # the state needs 16-byte alignment
    assert upd(C=FAKE + 5 * K + 4) == -1
    assert upd(x=FAKE + K + 1) == -1         # bf16 x misaligned
    assert upd(y=FAKE + 1024) == -1          # y inside the state
    assert upd(x=FAKE + 4096) == -1          # x inside the state
    assert upd(batch=0) == 0
    assert upd(headdim=0) == 0


def test_binding_has_no_cpu_path():
    from selective_state_space_39_b200 import ssm_scan_fwd
    x = torch.zeros(1, 4, 8)
    A = torch.zeros(8, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ssm_scan_fwd(x, x, A, torch.zeros(1, 4, 16), torch.zeros(1, 4, 16))


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "selective_state_space_39_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "ssm_oracle" not in text and "liboracle" not in text, f


@no_gpu_only
def test_oversized_problems_are_rejected(L):
    """Element counts past 2^40 are refused on the host (before any byte
    count could overflow), whatever the pointers."""
    p = bnd.ScanPlan()
    assert L.ssm_scan_plan(65535, 1 << 30, 1 << 24, 16, 1, ctypes.byref(p)) == -2
    assert L.ssm_scan_workspace_bytes(65535, 1 << 30, 1 << 24, 16, 1) == 0
    assert scan(L, batch=65535, seqlen=1 << 30, dim=1 << 20) == -2
    assert L.ssm_conv1d_silu_fwd(65535, 1 << 30, 1 << 20, 4, 1, FAKE, FAKE, None, 1, FAKE,
                                 None) == -2
    assert L.ssm_ssd_scan_fwd(65535, 1 << 30, 64, 64, 128, 1, FAKE, FAKE, FAKE, FAKE, FAKE,
                              None, None, 1, None, FAKE, None, None) == -2
    assert L.ssm_ssd_state_update(1 << 24, 1 << 20, 64, 128, 1, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  FAKE, None, None, 1, FAKE, None) == -2
    assert L.ssm_delta_sum(65535, 1 << 30, 1 << 20, 1, FAKE, None, 1, FAKE, None) == -2
    assert L.ssm_compose_carries(1 << 20, 65535, 1 << 20, 16, FAKE, None, FAKE, FAKE, FAKE,
                                 None) == -2


def test_noalloc_status_rejects_on_the_host(L):
    """ssm_scan_status_noalloc checks its sizes before it looks at any GPU:
    bad dtype or dstate, and problems the reserved scratch cannot hold."""
    assert L.ssm_scan_status_noalloc(1, 16, 64, 16, 7, None) == -2      # dtype
    assert L.ssm_scan_status_noalloc(1, 16, 64, 3, 1, None) == -2       # dstate
    assert L.ssm_scan_status_noalloc(-1, 16, 64, 16, 1, None) == -1     # size
    assert L.ssm_scan_status_noalloc(0, 16, 64, 16, 1, None) == 0       # empty: nothing ran
    os.environ["SSM_SCAN_SEGMENTS"] = "64"
    try:
        assert L.ssm_scan_status_noalloc(8, 4096, 2048, 16, 1, None) == -3
    finally:
        del os.environ["SSM_SCAN_SEGMENTS"]
