"""The timeout path of the bounded on-device waits, exercised without a real hang.

Test-only kernel instances (gdn_selftest.h) put a wait with a limit of zero polls
before any load, copy or MMA is issued.  The wait gives up, the status word in
the workspace records GDN_ERR_TIMEOUT, every CTA winds down without work, and the
call returns.  A normal call on the same stream and workspace afterwards must
match the oracle and leave the status word clear.  No GPU is faulted or hung.
"""
import ctypes

import pytest
import torch

from linear_attention_recurrence_rule_b200 import gdn
from linear_attention_recurrence_rule_b200.inputs import make_prefill, make_verify
from oracle import gdn_oracle as O
from parity_util import assert_close, to_dev

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _ptr(t):
    return None if t is None else P(t.data_ptr())


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def test_prefill_timeout_path_then_normal_call():
    lib = gdn.load_library()
    f = lib.gdn_selftest_prefill_timeout
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, P, P,
                  ctypes.c_size_t, P]
    x = make_prefill(2, 4, 128, 128, [200, 200], torch.bfloat16, seed=77)
    d = to_dev(x)
    N, T = 2, 200
    need = gdn.gdn_chunk_prefill_workspace_size(N, T, 2, 4, 128, 128, 64, gdn.GDN_BF16, 0)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(d["v"])
    hT = torch.empty(N, 4, 128, 128, device="cuda")
    rc = f(_ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]), _ptr(d["g"]), _ptr(d["beta"]), N, T, 2, 4,
           _ptr(o), _ptr(hT), _ptr(ws), need, _stream())
    assert rc == gdn.GDN_OK
    torch.cuda.synchronize()
    assert gdn.gdn_read_status(ws) == gdn.GDN_ERR_TIMEOUT
    # the same stream and workspace: a normal call clears the word and is exact again
    o2, h2 = gdn.gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], chunk=64,
                                   workspace=ws)
    torch.cuda.synchronize()
    assert gdn.gdn_read_status(ws) == gdn.GDN_OK
    o_ref, h_ref = O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"])
    assert_close(o2, o_ref, torch.bfloat16, "o after the timed-out call")
    assert_close(h2, h_ref, torch.bfloat16, "hT after the timed-out call")


def test_verify_timeout_path_then_normal_call():
    lib = gdn.load_library()
    f = lib.gdn_selftest_verify_timeout
    f.restype = ctypes.c_int
    f.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, ctypes.c_size_t, P]
    N, K, HK, HV = 6, 4, 2, 4
    x = make_verify(N, K, HK, HV, 128, 128, torch.bfloat16, seed=78, h0_std=0.2)
    d = to_dev(x)
    need = gdn.gdn_recurrent_verify_workspace_size(N, K, HV, 128)
    ws = torch.zeros(max(need, 1), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(d["v"])
    u = torch.empty(N, K, HV, 128, device="cuda")
    rc = f(_ptr(d["v"]), _ptr(d["state"]), N, K, HV, _ptr(o), _ptr(u), _ptr(ws), need, _stream())
    assert rc == gdn.GDN_OK
    torch.cuda.synchronize()
    assert gdn.gdn_read_status(ws) == gdn.GDN_ERR_TIMEOUT
    o2, _, u2 = gdn.gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                         rollback="deltas", workspace=ws)
    torch.cuda.synchronize()
    assert gdn.gdn_read_status(ws) == gdn.GDN_OK
    o_ref, _ = O.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    assert_close(o2, o_ref, torch.bfloat16, "o after the timed-out call")


def test_verify_tc_timeout_path_then_normal_call():
    """The tensor-core update-vector kernel (bf16, d = 128, up to 8 drafts)."""
    lib = gdn.load_library()
    f = lib.gdn_selftest_verify_tc_timeout
    f.restype = ctypes.c_int
    f.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, ctypes.c_size_t, P]
    N, K, HK, HV = 90, 6, 1, 2     # 180 heads: more than one per CTA
    x = make_verify(N, K, HK, HV, 128, 128, torch.bfloat16, seed=79, h0_std=0.2)
    d = to_dev(x)
    need = gdn.gdn_recurrent_verify_workspace_size(N, K, HV, 128)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(d["v"])
    u = torch.empty(N, K, HV, 128, device="cuda")
    rc = f(_ptr(d["v"]), _ptr(d["state"]), N, K, HV, _ptr(o), _ptr(u), _ptr(ws), need, _stream())
    assert rc == gdn.GDN_OK
    torch.cuda.synchronize()
    assert gdn.gdn_read_status(ws) == gdn.GDN_ERR_TIMEOUT
    o2, _, u2 = gdn.gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                         rollback="deltas", workspace=ws)
    torch.cuda.synchronize()
    assert gdn.gdn_read_status(ws) == gdn.GDN_OK
    o_ref, _ = O.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    assert_close(o2, o_ref, torch.bfloat16, "o after the timed-out call")
