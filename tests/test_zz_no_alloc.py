"""gdn_chunk_prefill_noalloc, the prefill for callers that cannot allocate device
memory (a fixed memory budget, no cudaMalloc on the hot path, or a host API
without a workspace), against the workspace-taking gdn_chunk_prefill.

Called through the C ABI directly.  Two calls in a row check that the scratch
the library keeps between calls (its status word) does not leak into the next
call's results.  Runs last so that a failure here does not hide other tests.
"""
import ctypes

import pytest
import torch

from linear_attention_recurrence_rule_b200 import gdn
from linear_attention_recurrence_rule_b200.inputs import make_prefill
from parity_util import assert_close, to_dev

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _noalloc_fn():
    lib = gdn.load_library()
    f = lib.gdn_chunk_prefill_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int, P, P, P]
    return f


def _ptr(t):
    return None if t is None else P(t.data_ptr())


@pytest.mark.parametrize("dtype,d,chunk", [(torch.bfloat16, 128, 64), (torch.float32, 32, 16)])
def test_noalloc_matches_workspace_entry_point(dtype, d, chunk):
    f = _noalloc_fn()
    x = make_prefill(2, 4, d, d, [300, 129], dtype, seed=2024, h0_std=0.05, packed=True)
    dv = to_dev(x)
    o_ref, h_ref = gdn.gdn_chunk_prefill(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"],
                                         h0=dv["h0"], cu_seqlens=dv["cu_seqlens"], chunk=chunk)
    torch.cuda.synchronize()
    o_ref64 = o_ref.double().cpu().numpy()
    h_ref64 = h_ref.double().cpu().numpy()
    N, T = 2, x["q"].shape[1]
    stream = P(torch.cuda.current_stream().cuda_stream)
    code = gdn.GDN_BF16 if dtype == torch.bfloat16 else gdn.GDN_F32
    for call in range(2):
        o = torch.full_like(dv["v"], float("nan"))
        hT = torch.full_like(dv["h0"], float("nan"))
        rc = f(_ptr(dv["q"]), _ptr(dv["k"]), _ptr(dv["v"]), _ptr(dv["g"]), _ptr(dv["beta"]),
               _ptr(dv["h0"]), _ptr(dv["cu_seqlens"]), N, T, 2, 4, d, d, chunk, 1.0, code,
               _ptr(o), _ptr(hT), stream)
        assert rc == gdn.GDN_OK, gdn.status_string(rc)
        torch.cuda.synchronize()
        # every on-device wait of the call completed (the status word in the library array)
        assert gdn.gdn_read_status(None) == gdn.GDN_OK
        assert_close(o, o_ref64, dtype, f"o, call {call}")
        assert_close(hT, h_ref64, dtype, f"hT, call {call}")
