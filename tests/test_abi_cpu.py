"""The C-ABI library loads, exports every symbol include/gdn.h declares, and its
host-side validation rejects bad arguments before anything reaches a GPU.
(No compute call is made here: every call below fails validation first.)"""
import ctypes
import glob
import os
import re

import pytest

from linear_attention_recurrence_rule_b200 import _build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return gdn.load_library()


def declared_symbols():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]*?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_two_calls():
    syms = declared_symbols()
    assert "gdn_chunk_prefill" in syms and "gdn_recurrent_step" in syms
    assert "gdn_chunk_prefill_workspace_size" in syms and "gdn_status_string" in syms
    assert "gdn_selftest_umma" in syms


def test_library_exports_every_declared_symbol(lib):
    handle = ctypes.CDLL(gdn.lib_path())
    for name in declared_symbols():
        assert hasattr(handle, name), f"{name} declared in gdn.h but not exported"


def test_library_is_sm100a_only():
    # the build command pins the one target architecture
    assert _build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings(lib):
    for code in range(7):
        s = gdn.status_string(code)
        assert isinstance(s, str) and s
    assert gdn.status_string(0) == "ok"
    assert lib.gdn_version() >= 100


P = ctypes.c_void_p


def fake(addr):
    return P(addr)  # never dereferenced: validation fails before any launch


def prefill_call(lib, **kw):
    a = dict(q=fake(0x1000), k=fake(0x2000), v=fake(0x3000), g=fake(0x4000), beta=fake(0x5000),
             h0=None, cu=None, N=1, T=64, HK=1, HV=2, dk=32, dv=32, chunk=16, scale=1.0,
             dtype=gdn.GDN_F32, o=fake(0x6000), hT=None, ws=None, ws_bytes=0)
    a.update(kw)
    return lib.gdn_chunk_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["h0"], a["cu"],
                                 a["N"], a["T"], a["HK"], a["HV"], a["dk"], a["dv"], a["chunk"],
                                 a["scale"], a["dtype"], a["o"], a["hT"], a["ws"], a["ws_bytes"],
                                 None)


def test_prefill_validation(lib):
    assert prefill_call(lib, q=None) == gdn.GDN_ERR_INVALID_ARG
    assert prefill_call(lib, o=None) == gdn.GDN_ERR_INVALID_ARG
    assert prefill_call(lib, HV=3, HK=2) == gdn.GDN_ERR_INVALID_ARG
    assert prefill_call(lib, N=-1) == gdn.GDN_ERR_INVALID_ARG
    assert prefill_call(lib, dtype=7) == gdn.GDN_ERR_INVALID_ARG
    assert prefill_call(lib, dk=48) == gdn.GDN_ERR_UNSUPPORTED
    assert prefill_call(lib, chunk=48) == gdn.GDN_ERR_UNSUPPORTED
    assert prefill_call(lib, dv=256) == gdn.GDN_ERR_UNSUPPORTED
    assert prefill_call(lib, q=fake(0x1004)) == gdn.GDN_ERR_ALIGNMENT
    assert prefill_call(lib, hT=fake(0x7008)) == gdn.GDN_ERR_ALIGNMENT
    # N == 0 is a valid empty problem: nothing is launched
    assert prefill_call(lib, N=0) == gdn.GDN_OK


def step_call(lib, **kw):
    a = dict(q=fake(0x1000), k=fake(0x2000), v=fake(0x3000), g=fake(0x4000), beta=fake(0x5000),
             state=fake(0x6000), N=2, HK=1, HV=2, dk=128, dv=128, scale=1.0,
             dtype=gdn.GDN_BF16, o=fake(0x7000))
    a.update(kw)
    return lib.gdn_recurrent_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state"], a["N"],
                                  a["HK"], a["HV"], a["dk"], a["dv"], a["scale"], a["dtype"],
                                  a["o"], None)


def test_step_validation(lib):
    assert step_call(lib, state=None) == gdn.GDN_ERR_INVALID_ARG
    assert step_call(lib, HK=3) == gdn.GDN_ERR_INVALID_ARG
    assert step_call(lib, dk=100) == gdn.GDN_ERR_UNSUPPORTED
    assert step_call(lib, dv=300) == gdn.GDN_ERR_UNSUPPORTED
    assert step_call(lib, state=fake(0x6004)) == gdn.GDN_ERR_ALIGNMENT
    assert step_call(lib, N=0) == gdn.GDN_OK


def test_workspace_size_rejects_bad_shapes(lib):
    assert gdn.gdn_chunk_prefill_workspace_size(1, 64, 2, 3, 128, 128, 64, gdn.GDN_BF16, 0) == 0
    assert gdn.gdn_chunk_prefill_workspace_size(-1, 64, 1, 2, 128, 128, 64, gdn.GDN_BF16, 0) == 0


def test_read_status_without_workspace(lib):
    # a NULL workspace reads the workspace-free prefill's library array on the
    # current device: without a usable device that is a CUDA error, not OK
    assert lib.gdn_read_status(None, 0, None) == gdn.GDN_ERR_CUDA


def verify_call(lib, **kw):
    a = dict(q=fake(0x1000), k=fake(0x2000), v=fake(0x3000), g=fake(0x4000), beta=fake(0x5000),
             state=fake(0x6000), N=2, K=4, HK=1, HV=2, dk=128, dv=128, scale=1.0,
             dtype=gdn.GDN_BF16, o=fake(0x7000), states=fake(0x8000), u=fake(0x9000))
    a.update(kw)
    return lib.gdn_recurrent_verify(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state"],
                                    a["N"], a["K"], a["HK"], a["HV"], a["dk"], a["dv"],
                                    a["scale"], a["dtype"], a["o"], a["states"], a["u"],
                                    a.get("pro", 0), a.get("ws", None), a.get("ws_bytes", 0),
                                    None)


def test_verify_validation(lib):
    assert verify_call(lib, o=None) == gdn.GDN_ERR_INVALID_ARG
    assert verify_call(lib, K=0) == gdn.GDN_ERR_INVALID_ARG
    assert verify_call(lib, HK=3) == gdn.GDN_ERR_INVALID_ARG
    assert verify_call(lib, K=17) == gdn.GDN_ERR_UNSUPPORTED   # above the draft limit
    assert verify_call(lib, dk=100) == gdn.GDN_ERR_UNSUPPORTED
    assert verify_call(lib, states=fake(0x8008)) == gdn.GDN_ERR_ALIGNMENT
    assert verify_call(lib, u=fake(0x9002)) == gdn.GDN_ERR_ALIGNMENT
    assert verify_call(lib, N=0) == gdn.GDN_OK
    # the update-vector form (no per-draft states) needs its workspace
    need = lib.gdn_recurrent_verify_workspace_size(2, 4, 2, 128)
    assert need == 16 + 2 * 2 * (2 * 4 * 128 + 2 * 16) * 4   # status word + tables
    assert verify_call(lib, states=None) == gdn.GDN_ERR_WORKSPACE
    assert verify_call(lib, states=None, ws=fake(0xa000), ws_bytes=need - 4) == gdn.GDN_ERR_WORKSPACE
    assert verify_call(lib, states=None, ws=fake(0xa008), ws_bytes=need) == gdn.GDN_ERR_ALIGNMENT
    assert lib.gdn_recurrent_verify_workspace_size(2, 17, 2, 128) == 0


def test_commit_validation(lib):
    def call(**kw):
        a = dict(states=fake(0x1000), acc=fake(0x2000), state=fake(0x3000), N=2, K=4, HV=2,
                 dk=128, dv=128)
        a.update(kw)
        return lib.gdn_state_commit(a["states"], a["acc"], a["state"], a["N"], a["K"], a["HV"],
                                    a["dk"], a["dv"], None)
    assert call(acc=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(K=0) == gdn.GDN_ERR_INVALID_ARG
    assert call(dk=3, dv=3) == gdn.GDN_ERR_UNSUPPORTED
    assert call(acc=fake(0x2002)) == gdn.GDN_ERR_ALIGNMENT
    assert call(N=0) == gdn.GDN_OK


def test_verify_and_commit_accept_empty_batch_with_null_buffers(lib):
    assert verify_call(lib, N=0, q=None, states=None) == gdn.GDN_OK
    assert lib.gdn_state_commit(None, None, None, 0, 4, 2, 128, 128, None) == gdn.GDN_OK


def test_commit_deltas_validation(lib):
    def call(**kw):
        a = dict(k=fake(0x1000), g=fake(0x2000), u=fake(0x3000), acc=fake(0x4000),
                 state=fake(0x5000), N=2, K=4, HK=1, HV=2, dk=128, dv=128, dtype=gdn.GDN_BF16)
        a.update(kw)
        return lib.gdn_state_commit_deltas(a["k"], a["g"], a["u"], a["acc"], a["state"], a["N"],
                                           a["K"], a["HK"], a["HV"], a["dk"], a["dv"], a["dtype"],
                                           a.get("pro", 0), None)
    assert call(u=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(HK=3) == gdn.GDN_ERR_INVALID_ARG
    assert call(dtype=9) == gdn.GDN_ERR_INVALID_ARG
    assert call(K=17) == gdn.GDN_ERR_UNSUPPORTED
    assert call(dv=300) == gdn.GDN_ERR_UNSUPPORTED
    assert call(state=fake(0x5004)) == gdn.GDN_ERR_ALIGNMENT
    assert call(N=0, k=None, u=None) == gdn.GDN_OK
    assert call(pro=16) == gdn.GDN_ERR_INVALID_ARG


def test_prologue_flags_are_validated(lib):
    assert gdn.PROLOGUE_ALL == gdn.PROLOGUE_NORM_Q | gdn.PROLOGUE_NORM_K | gdn.PROLOGUE_GATE_LOGITS
    text = "".join(open(h).read() for h in HEADERS)
    for name, val in (("NORM_Q", 1), ("NORM_K", 2), ("GATE_LOGITS", 4), ("ALL", 7)):
        assert re.search(rf"#define GDN_PROLOGUE_{name} {val}u", text)
    a = dict(q=fake(0x1000), k=fake(0x2000), v=fake(0x3000), g=fake(0x4000), beta=fake(0x5000))
    assert lib.gdn_chunk_prefill_ex(a["q"], a["k"], a["v"], a["g"], a["beta"], None, None, 1, 64,
                                    1, 2, 32, 32, 16, 1.0, gdn.GDN_F32, fake(0x6000), None, None,
                                    0, 16, None) == gdn.GDN_ERR_INVALID_ARG
    assert lib.gdn_recurrent_step_ex(a["q"], a["k"], a["v"], a["g"], a["beta"], fake(0x6000), 2,
                                     1, 2, 128, 128, 1.0, gdn.GDN_BF16, fake(0x7000), 16,
                                     None) == gdn.GDN_ERR_INVALID_ARG
    assert verify_call(lib, pro=16) == gdn.GDN_ERR_INVALID_ARG
    # one decay per value row: accepted by every call; unsupported shapes still rejected
    assert re.search(r"#define GDN_ROW_DECAY 8u", text)
    # (a supported shape would pass validation and launch: only rejected shapes here)
    assert lib.gdn_chunk_prefill_ex(a["q"], a["k"], a["v"], a["g"], a["beta"], None, None, 1, 64,
                                    1, 2, 48, 32, 16, 1.0, gdn.GDN_F32, fake(0x6000), None, None,
                                    0, gdn.ROW_DECAY, None) == gdn.GDN_ERR_UNSUPPORTED
    # the update-vector form with row decays passes the flag checks and stops at the
    # workspace check (nothing is launched here)
    assert verify_call(lib, states=None, ws=None, ws_bytes=0,
                       pro=gdn.ROW_DECAY) == gdn.GDN_ERR_WORKSPACE
    assert lib.gdn_recurrent_step_ex(a["q"], a["k"], a["v"], a["g"], a["beta"], fake(0x6004), 2,
                                     1, 2, 128, 128, 1.0, gdn.GDN_BF16, fake(0x7000),
                                     gdn.ROW_DECAY | 7, None) == gdn.GDN_ERR_ALIGNMENT
    # valid flags still go through the other checks first
    assert lib.gdn_recurrent_step_ex(a["q"], a["k"], a["v"], a["g"], a["beta"], fake(0x6004), 2,
                                     1, 2, 128, 128, 1.0, gdn.GDN_BF16, fake(0x7000), 7,
                                     None) == gdn.GDN_ERR_ALIGNMENT


def test_commit_verify_validation(lib):
    def call(**kw):
        a = dict(pk=fake(0x1000), pg=fake(0x2000), pu=fake(0x3000), acc=fake(0x4000), Kp=4,
                 q=fake(0x5000), k=fake(0x6000), v=fake(0x7000), g=fake(0x8000),
                 beta=fake(0x9000), state=fake(0xa000), N=2, K=4, HK=1, HV=2, dk=128, dv=128,
                 dtype=gdn.GDN_BF16, o=fake(0xb000), u=fake(0xc000), pro=0, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.gdn_recurrent_commit_verify(
            a["pk"], a["pg"], a["pu"], a["acc"], a["Kp"], a["q"], a["k"], a["v"], a["g"],
            a["beta"], a["state"], a["N"], a["K"], a["HK"], a["HV"], a["dk"], a["dv"], 1.0,
            a["dtype"], a["o"], a["u"], a["pro"], a["ws"], a["ws_bytes"], None)
    # every call below is rejected before anything is enqueued
    assert call(Kp=0) == gdn.GDN_ERR_INVALID_ARG
    assert call(pu=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(pro=16) == gdn.GDN_ERR_INVALID_ARG
    assert call(Kp=17) == gdn.GDN_ERR_UNSUPPORTED
    assert call(pro=gdn.ROW_DECAY) == gdn.GDN_ERR_WORKSPACE   # row decays accepted
    assert call(pk=fake(0x1008)) == gdn.GDN_ERR_ALIGNMENT
    assert call() == gdn.GDN_ERR_WORKSPACE
    need = lib.gdn_recurrent_commit_verify_workspace_size(2, 4, 4, 2, 128)
    assert need == 16 + 2 * 2 * ((2 * 4 * 128 + 2 * 16) + (4 * 128 + 4)) * 4
    assert call(ws=fake(0xd000), ws_bytes=need - 16) == gdn.GDN_ERR_WORKSPACE
    assert call(ws=fake(0xd008), ws_bytes=need) == gdn.GDN_ERR_ALIGNMENT
    assert call(N=0, q=None, pk=None) == gdn.GDN_OK


# ---- the layer steps (short convolution, output gate); fake pointers never reach a launch
def conv_call(lib, **kw):
    a = dict(x=fake(0x1000), w=fake(0x2000), b=None, cs=None, cu=None, N=1, T=64, C=64, W=4,
             flags=0, dtype=gdn.GDN_BF16, y=fake(0x3000))
    a.update(kw)
    return lib.gdn_short_conv(a["x"], a["w"], a["b"], a["cs"], a["cu"], a["N"], a["T"], a["C"],
                              a["W"], a["flags"], a["dtype"], a["y"], None)


def test_short_conv_validation(lib):
    assert conv_call(lib, flags=32) == gdn.GDN_ERR_INVALID_ARG
    assert conv_call(lib, x=None) == gdn.GDN_ERR_INVALID_ARG
    assert conv_call(lib, w=None) == gdn.GDN_ERR_INVALID_ARG
    assert conv_call(lib, y=None) == gdn.GDN_ERR_INVALID_ARG
    assert conv_call(lib, N=-1) == gdn.GDN_ERR_INVALID_ARG
    assert conv_call(lib, C=0) == gdn.GDN_ERR_INVALID_ARG
    assert conv_call(lib, dtype=7) == gdn.GDN_ERR_INVALID_ARG
    assert conv_call(lib, W=1) == gdn.GDN_ERR_UNSUPPORTED
    assert conv_call(lib, W=gdn.CONV_MAX_WIDTH + 1) == gdn.GDN_ERR_UNSUPPORTED
    assert conv_call(lib, C=12) == gdn.GDN_ERR_UNSUPPORTED                 # bf16: 8 per vector
    assert conv_call(lib, C=12, dtype=gdn.GDN_F32, x=fake(0x1008)) == gdn.GDN_ERR_ALIGNMENT
    assert conv_call(lib, cs=fake(0x4004)) == gdn.GDN_ERR_ALIGNMENT
    assert conv_call(lib, w=fake(0x2004)) == gdn.GDN_ERR_ALIGNMENT
    assert conv_call(lib, N=0) == gdn.GDN_OK                                # empty batch


def test_output_gate_validation(lib):
    def call(o=fake(0x1000), z=fake(0x2000), rows=4, C=64, dtype=gdn.GDN_F32):
        return lib.gdn_output_gate(o, z, rows, C, dtype, None)
    assert call(o=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(z=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(rows=-1) == gdn.GDN_ERR_INVALID_ARG
    assert call(C=0) == gdn.GDN_ERR_INVALID_ARG
    assert call(dtype=5) == gdn.GDN_ERR_INVALID_ARG
    assert call(rows=1, C=3) == gdn.GDN_ERR_UNSUPPORTED
    assert call(z=fake(0x2004)) == gdn.GDN_ERR_ALIGNMENT
    assert call(rows=0) == gdn.GDN_OK


def step_layer_call(lib, **kw):
    a = dict(q=fake(0x1000), k=fake(0x2000), v=fake(0x3000), g=fake(0x4000), beta=fake(0x5000),
             state=fake(0x6000), w=fake(0x7000), b=None, cs=fake(0x8000), W=4, z=fake(0x9000),
             N=2, HK=1, HV=2, dk=64, dv=64, dtype=gdn.GDN_BF16, o=fake(0xa000), flags=0)
    a.update(kw)
    return lib.gdn_recurrent_step_layer(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state"],
                                        a["w"], a["b"], a["cs"], a["W"], a["z"], a["N"], a["HK"],
                                        a["HV"], a["dk"], a["dv"], 1.0, a["dtype"], a["o"],
                                        a["flags"], None)


def test_step_layer_validation(lib):
    assert step_layer_call(lib, flags=32) == gdn.GDN_ERR_INVALID_ARG
    assert step_layer_call(lib, o=None) == gdn.GDN_ERR_INVALID_ARG
    assert step_layer_call(lib, cs=None) == gdn.GDN_ERR_INVALID_ARG         # conv without state
    assert step_layer_call(lib, W=1) == gdn.GDN_ERR_UNSUPPORTED
    assert step_layer_call(lib, W=9) == gdn.GDN_ERR_UNSUPPORTED
    assert step_layer_call(lib, dk=48) == gdn.GDN_ERR_UNSUPPORTED
    assert step_layer_call(lib, z=fake(0x9001)) == gdn.GDN_ERR_ALIGNMENT     # bf16: 2-byte
    assert step_layer_call(lib, cs=fake(0x8001)) == gdn.GDN_ERR_ALIGNMENT
    assert step_layer_call(lib, q=fake(0x1008)) == gdn.GDN_ERR_ALIGNMENT
    assert step_layer_call(lib, N=0) == gdn.GDN_OK
    assert step_layer_call(lib, N=0, w=None, cs=None, z=None,
                           flags=gdn.PROLOGUE_ALL | gdn.ROW_DECAY | gdn.CONV_SILU) == gdn.GDN_OK


def prefill_layer_call(lib, **kw):
    a = dict(q=fake(0x1000), k=fake(0x2000), v=fake(0x3000), g=fake(0x4000), beta=fake(0x5000),
             N=1, T=64, HK=1, HV=2, dk=32, dv=32, chunk=16, dtype=gdn.GDN_F32, o=fake(0x6000),
             w=fake(0x7000), b=None, cs=None, W=4, z=None, flags=0, ws=None, ws_bytes=0)
    a.update(kw)
    return lib.gdn_chunk_prefill_layer(a["q"], a["k"], a["v"], a["g"], a["beta"], None, None,
                                       a["N"], a["T"], a["HK"], a["HV"], a["dk"], a["dv"],
                                       a["chunk"], 1.0, a["dtype"], a["o"], None, a["w"], a["b"],
                                       a["cs"], a["W"], a["z"], a["flags"], a["ws"], a["ws_bytes"],
                                       None)


def test_prefill_layer_validation(lib):
    assert prefill_layer_call(lib, flags=32) == gdn.GDN_ERR_INVALID_ARG
    assert prefill_layer_call(lib, q=None) == gdn.GDN_ERR_INVALID_ARG
    assert prefill_layer_call(lib, dk=48) == gdn.GDN_ERR_UNSUPPORTED
    assert prefill_layer_call(lib, W=9) == gdn.GDN_ERR_UNSUPPORTED
    assert prefill_layer_call(lib, z=fake(0x9008)) == gdn.GDN_ERR_ALIGNMENT
    # the convolved values need workspace: none given
    assert prefill_layer_call(lib) == gdn.GDN_ERR_WORKSPACE
    need = lib.gdn_chunk_prefill_layer_workspace_size(1, 64, 1, 2, 32, 32, 16, gdn.GDN_F32, 0, 1, 0)
    assert need >= 64 * 2 * 32 * 4
    assert prefill_layer_call(lib, ws=fake(0x10000), ws_bytes=need - 1) == gdn.GDN_ERR_WORKSPACE
    assert prefill_layer_call(lib, ws=fake(0x10008), ws_bytes=need) == gdn.GDN_ERR_ALIGNMENT
    assert prefill_layer_call(lib, N=0) == gdn.GDN_OK
    assert lib.gdn_chunk_prefill_layer_workspace_size(1, 64, 1, 2, 32, 32, 16, gdn.GDN_F32, 0, 0, 0) == 0
    # the gate factors: fp16, one per output element
    assert lib.gdn_chunk_prefill_layer_workspace_size(1, 64, 1, 2, 32, 32, 16, gdn.GDN_F32, 0, 0,
                                                      1) >= 64 * 2 * 32 * 2
    assert prefill_layer_call(lib, w=None, z=fake(0x9000)) == gdn.GDN_ERR_WORKSPACE
