"""Host-side argument checks of the C ABI (CPU only, no compute call).

Every case here is one the library must reject before it touches the device, so the
fake, never dereferenced pointer values below are safe anywhere: include/gtr_gla.h
states the checks (null or misaligned buffers, sizes out of range, an unknown
direction, an output that overlaps an input, int32 overflow of the element counts).
"""
import ctypes

import pytest

from recurrent_vision_backbone_b200 import build, gla

MB = 1 << 24   # fake buffers 16 MiB apart, 16-byte aligned


@pytest.fixture(scope="module")
def lib():
    return gla.load(build.build())


def call(lib, entry="gtr_gla_fwd", q=1, k=2, v=3, g=4, out=5, B=1, heads=2, H=8, W=8, dk=64, dv=64,
         direction=0, chunk=64, s0=None, sf=None):
    P = lambda x: None if x is None else ctypes.c_void_p(x * MB if x < 64 else x)
    args = [P(q), P(k), P(v), P(g), B, heads, H, W, dk, dv, direction, chunk, P(s0), P(out), P(sf)]
    if entry == "gtr_gla_fwd_ws":
        return getattr(lib, entry)(*args, P(6), ctypes.c_size_t(1 << 20), None)
    return getattr(lib, entry)(*args, None)


@pytest.mark.parametrize("entry", ["gtr_gla_fwd", "gtr_gla_fwd_ws", "gtr_gla_fwd_static"])
@pytest.mark.parametrize("bad, want", [
    (dict(B=0), "invalid"), (dict(heads=-1), "invalid"), (dict(H=-1), "invalid"),
    (dict(dk=0), "invalid"), (dict(q=None), "invalid"), (dict(out=None), "invalid"),
    (dict(direction=4), "invalid"), (dict(direction=-1), "invalid"), (dict(chunk=0), "invalid"),
    (dict(chunk=32), "unsupported"), (dict(dk=96), "unsupported"), (dict(dv=96), "unsupported"),
    (dict(q=1 * MB + 8), "invalid"),                 # misaligned input
    (dict(s0=7 * MB + 4), "invalid"),                # misaligned initial state
    (dict(out=1 * MB + 64), "invalid"),              # output overlaps q
    (dict(out=3 * MB), "invalid"),                   # output is v
    (dict(H=46341, W=46341), "invalid"),             # N beyond int32
    (dict(B=4096, heads=64, H=128, W=128), "invalid"),  # B*N*heads*dk beyond int32
])
def test_rejected_before_any_device_work(lib, entry, bad, want):
    code = {"invalid": gla.GTR_ERR_INVALID_ARG, "unsupported": gla.GTR_ERR_UNSUPPORTED}[want]
    assert call(lib, entry, **bad) == code


def call_bwd(lib, q=1, k=2, v=3, g=4, do=5, s0=None, dsf=None, B=1, heads=2, H=8, W=8, dk=64, dv=64,
             direction=0, chunk=64, gq=6, gk=7, gv=8, gg=9, gs=None, ws=10, ws_bytes=1 << 22):
    P = lambda x: None if x is None else ctypes.c_void_p(x * MB if x < 64 else x)
    return lib.gtr_gla_bwd(P(q), P(k), P(v), P(g), P(do), P(s0), P(dsf), B, heads, H, W, dk, dv, direction,
                           chunk, P(gq), P(gk), P(gv), P(gg), P(gs), P(ws), ctypes.c_size_t(ws_bytes), None)


@pytest.mark.parametrize("bad, want", [
    (dict(B=0), "invalid"), (dict(direction=4), "invalid"), (dict(chunk=0), "invalid"),
    (dict(chunk=32), "unsupported"), (dict(dk=96), "unsupported"), (dict(dv=128), "unsupported"),
    (dict(do=None), "invalid"), (dict(gg=None), "invalid"),
    (dict(gq=6 * MB + 4), "invalid"),             # misaligned gradient
    (dict(gv=5), "invalid"),                       # grad_v is d_out
    (dict(gk=6 * MB + 64), "invalid"),             # grad_k overlaps grad_q
    (dict(gs=1), "invalid"),                       # grad_init_state overlaps q
    (dict(ws=None), "invalid"),                    # no workspace
    (dict(ws_bytes=4096), "invalid"),              # short workspace
    (dict(ws=10 * MB + 128), "invalid"),           # workspace not 256-byte aligned
    (dict(ws=7 * MB + 256), "invalid"),            # workspace overlaps grad_k
    (dict(ws=3 * MB), "invalid"),                  # workspace is v
    (dict(H=46341, W=46341), "invalid"),           # N beyond int32
])
def test_backward_rejected_before_any_device_work(lib, bad, want):
    code = {"invalid": gla.GTR_ERR_INVALID_ARG, "unsupported": gla.GTR_ERR_UNSUPPORTED}[want]
    assert call_bwd(lib, **bad) == code


def test_backward_workspace_size(lib):
    # two 64 x 64 fp32 tiles and two 64-float vectors per (sequence, chunk), 64 floats per
    # sequence, each part rounded up to 256 bytes; 0 for rejected shapes or an empty grid
    n_seq, nc = 2 * 16, 25
    want = 2 * n_seq * nc * 16384 + 2 * ((n_seq * nc * 256 + 255) // 256 * 256) + n_seq * 256
    assert gla.bwd_workspace_bytes(2, 16, 40, 40, 64, 64) == want
    assert gla.bwd_workspace_bytes(2, 16, 40, 40, 128, 64) == want   # one key half, reused
    assert gla.bwd_workspace_bytes(2, 16, 40, 40, 64, 128) == 0
    assert gla.bwd_workspace_bytes(2, 16, 0, 40, 64, 64) == 0
