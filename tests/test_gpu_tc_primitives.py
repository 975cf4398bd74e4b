"""tcgen05 / TMA building blocks against plain matrix products (one CTA), in the
exact operand layouts the tensor-core prefill uses."""
import ctypes

import pytest
import torch

from linear_attention_recurrence_rule_b200 import gdn

pytestmark = pytest.mark.gpu


def test_umma_operand_patterns():
    lib = gdn.load_library()
    f = lib.gdn_selftest_umma
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 15
    g = torch.Generator().manual_seed(0)
    r = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    X, Y, Z, R, U, S, W = r(128, 128), r(64, 128), r(64, 128), r(64, 64), r(128, 64), \
        r(128, 128), r(128, 64)
    D0 = torch.randn(128, 64, generator=g)
    dev = [t.cuda() for t in (X, Y, Z, R, U, S, W, D0)]
    outs = [torch.full((128, 64), float("nan"), device="cuda"),
            torch.full((128, 64), float("nan"), device="cuda"),
            torch.full((128, 128), float("nan"), device="cuda"),
            torch.full((128, 64), float("nan"), device="cuda"),
            torch.full((128, 128), float("nan"), device="cuda")]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = f(*[ctypes.c_void_p(t.data_ptr()) for t in dev + outs + [status]],
           ctypes.c_void_p(stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "an on-device wait timed out"
    d = lambda t: t.double()
    refs = [d(X) @ d(Y).T, d(Z).T @ d(R).T, d(U) @ d(Z), d(D0) - d(S) @ d(W), d(U) @ d(Z)]
    for name, out, ref in zip(("X Y^T", "Z^T R^T", "U Z", "D0 - S W", "U(tmem) Z"), outs, refs):
        err = (out.double().cpu() - ref).abs().max().item()
        assert err < 1e-3, f"{name}: max|err| {err}"
