"""Host-side tests of the C-ABI library (no GPU needed): it loads, exports every function the
header declares, and its validation / size queries follow the documented rules.  No call here
reaches a CUDA runtime function."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lrscan.h")


@pytest.fixture(scope="module")
def L():
    from selective_state_space_09_b200 import build
    build.build()
    from selective_state_space_09_b200 import lrscan
    return lrscan


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(lr_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["lr_scan_fwd", "lr_scan_bwd", "lr_ckpt_bytes", "lr_workspace_bytes",
              "lr_get_error", "lr_status_string", "lr_last_dispatch", "lr_validate"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    so = ctypes.CDLL(L.LIB_PATH)
    for n in declared_functions():
        assert hasattr(so, n), n


def test_status_strings(L):
    for s, want in enumerate(L.STATUS):
        assert L.lib.lr_status_string(s).decode() == want
    assert L.lib.lr_version() == 1


def _ok(lrs, **kw):
    return lrs.validate(lrs.make_desc(**kw))


def test_validation_rules(L):
    import torch
    f32, bf = torch.float32, torch.bfloat16
    assert _ok(L, kind="rglru", io=f32, B=1, L=1024, D=256, segment=128) == 0
    assert _ok(L, kind="rglru", io=f32, B=1, L=1, D=4, segment=1) == 0
    assert _ok(L, kind="rglru", io=f32, B=1, L=10, D=3, segment=4) == 3        # 12 B rows
    assert _ok(L, kind="rglru", io=f32, B=0, L=10, D=4, segment=4) == 1
    assert _ok(L, kind="rglru", io=f32, B=1, L=10, D=4, segment=0) == 1
    assert _ok(L, kind="rglru", io=f32, B=1, L=1000, D=4, segment=512) == 2    # S > 256
    assert _ok(L, kind="rglru", io=f32, B=1, L=10, D=4, segment=4, disc="zoh") == 1
    assert _ok(L, kind="rotlru", io=f32, B=16, L=16384, D=4096, segment=256) == 0
    assert _ok(L, kind="rotlru", io=f32, B=1, L=8, D=5, segment=4) == 1        # odd D
    assert _ok(L, kind="rotlru", io=f32, B=1, L=8, D=4, segment=4) == 3        # g rows 8 B
    # kinds whose kernels a build lacks report UNSUPPORTED (2) for otherwise valid requests
    assert _ok(L, kind="s6", io=bf, B=8, L=2048, D=2048, N=16, segment=64, disc="zoh") == 0
    assert _ok(L, kind="s6", io=bf, B=8, L=2048, D=2048, N=16, segment=256, disc="zoh") == 2
    assert _ok(L, kind="s6", io=bf, B=8, L=2048, D=2048, N=8, segment=64, disc="zoh") == 2
    assert _ok(L, kind="s6", io=f32, B=8, L=2048, D=2048, N=16, segment=64, disc="zoh") == 2
    assert _ok(L, kind="s6", io=bf, B=8, L=2048, D=2048, N=16, segment=256) == 1  # no disc
    assert _ok(L, kind="ssd", io=bf, B=2, L=4096, H=32, P=64, N=128, G=1, segment=128,
               chunk=128, disc="zoh") == 0
    assert _ok(L, kind="ssd", io=bf, B=2, L=4096, H=32, P=64, N=128, G=1, segment=256,
               chunk=64, disc="zoh") == 2                                        # chunk != 128
    assert _ok(L, kind="ssd", io=bf, B=2, L=4096, H=32, P=64, N=128, G=1, segment=128,
               disc="bilinear") == 0                                             # signed decays
    assert _ok(L, kind="ssd", io=bf, B=2, L=64, H=32, P=64, N=128, G=3, segment=64,
               disc="zoh") == 1                                                  # H % G
    assert _ok(L, kind="gla", io=bf, B=4, L=2048, H=16, P=128, N=128, segment=128, chunk=128) == 0
    assert _ok(L, kind="gla", io=bf, B=4, L=2048, H=16, P=96, N=128, segment=128) == 2
    assert _ok(L, kind="gla", io=bf, B=4, L=2048, H=16, P=128, N=128, segment=256,
               disc="zoh") == 1


def test_size_queries(L):
    import torch
    d = L.make_desc("rotlru", torch.float32, B=16, L=16384, D=4096, segment=256)
    assert L.ckpt_bytes(d) == 64 * 16 * 4096 * 4                    # 16 MiB of checkpoints
    assert L.workspace_bytes(d, False) > 256 and L.workspace_bytes(d, True) > 256
    d = L.make_desc("rglru", torch.float32, B=1, L=1000, D=256, segment=128)
    assert L.ckpt_bytes(d) == 8 * 1 * 256 * 4                       # ceil(1000/128) = 8
    bad = L.make_desc("rglru", torch.float32, B=1, L=1000, D=3, segment=128)
    assert L.ckpt_bytes(bad) == 0 and L.workspace_bytes(bad, True) == 0
    # SSD / GLA: one chunk per segment keeps a bf16 tile copy beside every f32 state; longer
    # segments (whole chunks) keep the f32 segment states only
    bf = torch.bfloat16
    ssd = dict(kind="ssd", io=bf, B=2, L=4096, H=32, P=64, N=128, G=1, chunk=128, disc="zoh")
    state = 2 * 32 * 128 * 64
    assert L.ckpt_bytes(L.make_desc(segment=128, **ssd)) == 32 * state * 6
    assert L.ckpt_bytes(L.make_desc(segment=256, **ssd)) == 16 * state * 4
    assert L.ckpt_bytes(L.make_desc(segment=512, **ssd)) == 8 * state * 4
    assert L.validate(L.make_desc(segment=192, **ssd)) == 2          # not a whole number of chunks
    gla = dict(kind="gla", io=bf, B=4, L=2048, H=16, P=128, N=128, chunk=128)
    assert L.ckpt_bytes(L.make_desc(segment=256, **gla)) == 8 * 4 * 16 * 128 * 128 * 4


def test_calls_rejected_before_any_launch(L):
    """Invalid requests return their status from host-side validation (no CUDA call made)."""
    import torch
    d = L.make_desc("rglru", torch.float32, B=1, L=16, D=32, segment=8)
    ii = L.Inputs()  # all NULL
    s = L.lib.lr_scan_fwd(ctypes.byref(d), ctypes.byref(ii), None, None, None, 0, None)
    assert s == 1
    bad = L.make_desc("rglru", torch.float32, B=1, L=16, D=6, segment=8)
    s = L.lib.lr_scan_fwd(ctypes.byref(bad), ctypes.byref(ii), None, None, None, 0, None)
    assert s == 3
    # misaligned pointer
    ii = L.Inputs(a=ctypes.c_void_p(0x1004), b=ctypes.c_void_p(0x2000))
    s = L.lib.lr_scan_fwd(ctypes.byref(d), ctypes.byref(ii), ctypes.c_void_p(0x3000),
                          ctypes.c_void_p(0x4000), ctypes.c_void_p(0x5000), 1 << 20, None)
    assert s == 3
    # workspace too small
    ii = L.Inputs(a=ctypes.c_void_p(0x1000), b=ctypes.c_void_p(0x2000))
    s = L.lib.lr_scan_fwd(ctypes.byref(d), ctypes.byref(ii), ctypes.c_void_p(0x3000),
                          ctypes.c_void_p(0x4000), ctypes.c_void_p(0x5000), 16, None)
    assert s == 4
    assert L.last_launch_count() == 0


def test_step_calls_rejected_before_any_launch(L):
    """lr_step's host-side checks: missing pointers, misalignment, the limits of the step path."""
    import torch
    V = ctypes.c_void_p
    d = L.make_desc("rglru", torch.float32, B=2, L=1, D=32)
    ok = L.Inputs(a=V(0x1000), b=V(0x2000))
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(ok), None, None, V(0x3000), None) == 1  # no state_out
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(L.Inputs()), None, V(0x4000), V(0x3000), None) == 1
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(ok), V(0x1002), V(0x4000), V(0x3000), None) == 3
    bad = L.Inputs(a=V(0x1001), b=V(0x2000))
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(bad), None, V(0x4000), V(0x3000), None) == 3
    # rotlru b and y are read as (re, im) pairs: two elements of alignment
    d = L.make_desc("rotlru", torch.float32, B=1, L=1, D=8)
    ii = L.Inputs(b=V(0x1004), g=V(0x2000), mag=V(0x3000), theta=V(0x3100))
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(ii), None, V(0x4000), V(0x5000), None) == 3
    # limits of the step path: S6 N <= 32, SSD / GLA N <= 128; SSD heads divisible by groups
    s6in = L.Inputs(x=V(0x1000), delta=V(0x2000), A=V(0x3000), Bm=V(0x4000), Cm=V(0x5000))
    d = L.make_desc("s6", torch.bfloat16, B=1, L=1, D=8, N=64, disc="zoh")
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(s6in), None, V(0x6000), V(0x7000), None) == 2
    d = L.make_desc("ssd", torch.bfloat16, B=1, L=1, H=4, P=8, N=256, G=1, disc="zoh")
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(s6in), None, V(0x6000), V(0x7000), None) == 2
    d = L.make_desc("ssd", torch.bfloat16, B=1, L=1, H=4, P=8, N=16, G=3, disc="zoh")
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(s6in), None, V(0x6000), V(0x7000), None) == 1
    d = L.make_desc("gla", torch.bfloat16, B=1, L=1, H=2, P=8, N=16, disc="zoh")
    gin = L.Inputs(q=V(0x1000), k=V(0x2000), v=V(0x3000), g=V(0x4000))
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(gin), None, V(0x6000), V(0x7000), None) == 1
    assert L.last_launch_count() == 0


def test_rglru_gates_rules(L):
    """LR_RGLRU_GATES: rglru f32 only, not with the full-state mode; a scan call without x or
    Lambda, and an lr_rglru_fwd_noalloc call with the flag, are rejected before any launch; the
    backward workspace holds the per-tile dLambda partials."""
    import torch
    V = ctypes.c_void_p

    def gated(kind="rglru", io=torch.float32, **kw):
        d = L.make_desc(kind, io, **kw)
        d.flags |= L.RGLRU_GATES
        return d
    assert L.validate(gated(B=1, L=1024, D=256, segment=128)) == 0
    assert L.validate(gated(io=torch.bfloat16, B=1, L=64, D=64, segment=16)) == 2
    d = gated(B=1, L=64, D=64, segment=16)
    d.flags |= L.FULL_STATE
    assert L.validate(d) == 2
    assert L.validate(gated("rotlru", B=1, L=64, D=64, segment=16)) == 1
    assert L.validate(gated("s6", io=torch.bfloat16, B=1, L=64, D=64, N=16, segment=16, disc="zoh")) == 1
    d = gated(B=1, L=64, D=64, segment=16)
    plain = L.make_desc("rglru", torch.float32, B=1, L=64, D=64, segment=16)
    assert L.workspace_bytes(d, False) == L.workspace_bytes(plain, False)
    assert L.workspace_bytes(d, True) >= L.workspace_bytes(plain, True) + 8 * 4 * 64
    no_x = L.Inputs(a=V(0x1000), b=V(0x2000), A=V(0x3000))
    assert L.lib.lr_scan_fwd(ctypes.byref(d), ctypes.byref(no_x), V(0x4000), V(0x5000), V(0x6000), 1 << 20,
                             None) == 1
    no_lam = L.Inputs(a=V(0x1000), b=V(0x2000), x=V(0x3000))
    assert L.lib.lr_step(ctypes.byref(d), ctypes.byref(no_lam), None, V(0x4000), V(0x5000), None) == 1
    so = ctypes.CDLL(L.LIB_PATH)
    so.lr_rglru_fwd_noalloc.restype = ctypes.c_int
    assert so.lr_rglru_fwd_noalloc(ctypes.byref(d), V(0x1000), V(0x2000), V(0x3000), V(0x4000), None, 0) == 2
    assert L.last_launch_count() == 0


def test_plan_buffers_cover_the_queried_sizes(L):
    import torch
    for d in (L.make_desc("rotlru", torch.float32, B=2, L=1000, D=64, segment=64),
              L.make_desc("rglru", torch.bfloat16, B=3, L=77, D=96, segment=16)):
        p = L.Plan(d, "cpu")
        assert p.ws_bytes >= max(L.workspace_bytes(d, False), L.workspace_bytes(d, True))
        assert p.ckpt.numel() * 4 >= L.ckpt_bytes(d)
        assert p.ckpt_view().shape[0] == (d.L + d.segment - 1) // d.segment


def test_every_gpu_test_case_passes_host_validation(L):
    """The descriptors of the GPU parity cases are valid for the library (checked on the CPU, so a
    shape-rule mistake does not cost a GPU run)."""
    import torch
    import test_gpu_diag as gd
    import test_gpu_s6 as gs
    import test_gpu_chunk as gc
    f32, bf = torch.float32, torch.bfloat16
    for B, Lq, D, S, io in gd.RGLRU_CASES:
        assert _ok(L, kind="rglru", io=f32 if io == "f32" else bf, B=B, L=Lq, D=D, segment=S) == 0
    for B, Lq, D, S, io in gd.ROTLRU_CASES:
        assert _ok(L, kind="rotlru", io=f32 if io == "f32" else bf, B=B, L=Lq, D=D, segment=S) == 0
    for B, Lq, D, S, disc, wz, wd in gs.CASES:
        assert _ok(L, kind="s6", io=bf, B=B, L=Lq, D=D, N=16, segment=S, disc=disc, has_z=wz, has_d=wd) == 0
    for B, Lq, H, P, G in gc.SSD_CASES:
        assert _ok(L, kind="ssd", io=bf, B=B, L=Lq, H=H, P=P, N=128, G=G, segment=128, chunk=128,
                   disc="zoh", has_d=True) == 0
    for disc in ("dirac", "zoh_euler", "bilinear"):  # bilinear: signed decays (log magnitude + parity)
        for hz in (False, True):
            assert _ok(L, kind="ssd", io=bf, B=1, L=512, H=4, P=64, N=128, G=1, segment=128, chunk=128,
                       disc=disc, has_d=True, has_z=hz) == 0
    for B, Lq, H, V in gc.GLA_CASES:
        assert _ok(L, kind="gla", io=bf, B=B, L=Lq, H=H, P=V, N=128, segment=128, chunk=128) == 0
