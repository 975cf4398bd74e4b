"""gdn_chunk_prefill_host (host-resident inputs and outputs, streamed in segments)
against gdn_chunk_prefill on the device and against the oracle."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_rule_b200 import gdn
from linear_attention_recurrence_rule_b200.inputs import make_prefill
from oracle import gdn_oracle as O
from parity_util import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _host(x):
    return {k: (v.pin_memory() if isinstance(v, torch.Tensor) and k != "cu_seqlens" else v)
            for k, v in x.items()}


@pytest.mark.parametrize("dtype,d,chunk", [(torch.bfloat16, 128, 64), (torch.float32, 32, 16)])
def test_host_prefill_bitwise_equals_device_prefill(dtype, d, chunk):
    # segments that are multiples of the chunk reproduce the one-call result bit for bit
    x = make_prefill(2, 4, d, d, [700, 700], dtype, seed=77, h0_std=0.05, packed=False)
    dv = to_dev(x)
    o_ref, h_ref = gdn.gdn_chunk_prefill(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"],
                                         h0=dv["h0"], chunk=chunk)
    hx = _host(x)
    o, hT = gdn.gdn_chunk_prefill_host(hx["q"], hx["k"], hx["v"], hx["g"], hx["beta"],
                                       h0=dv["h0"].clone(), chunk=chunk, segment=4 * chunk)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref.cpu())
    assert torch.equal(hT, h_ref)


@pytest.mark.parametrize("segment", [100, 257, 0])
def test_host_prefill_matches_oracle_any_segment(segment):
    # a segment that is not a multiple of the chunk only moves chunk boundaries
    x = make_prefill(1, 2, 128, 128, [1500], torch.bfloat16, seed=78, h0_std=0.05, packed=False)
    hx = _host(x)
    h0 = x["h0"].cuda()
    o, hT = gdn.gdn_chunk_prefill_host(hx["q"], hx["k"], hx["v"], hx["g"], hx["beta"], h0=h0,
                                       segment=segment)
    torch.cuda.synchronize()
    o_ref, h_ref = O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], h0=x["h0"])
    assert_close(o[0], o_ref, torch.bfloat16, "o")
    assert_close(hT, h_ref, torch.bfloat16, "hT")


def test_host_prefill_state_aliasing_and_no_final_state():
    x = make_prefill(1, 2, 128, 128, [640], torch.bfloat16, seed=79, h0_std=0.05, packed=False)
    hx = _host(x)
    h = x["h0"].cuda()
    o1, _ = gdn.gdn_chunk_prefill_host(hx["q"], hx["k"], hx["v"], hx["g"], hx["beta"], h0=h,
                                       hT=h, segment=128)              # hT aliases h0
    o2, none = gdn.gdn_chunk_prefill_host(hx["q"], hx["k"], hx["v"], hx["g"], hx["beta"],
                                          h0=x["h0"].cuda(), segment=192,
                                          output_final_state=False)
    torch.cuda.synchronize()
    assert none is None
    _, h_ref = O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], h0=x["h0"])
    assert_close(h, h_ref, torch.bfloat16, "hT (aliased)")
    assert torch.equal(o1, o2)


def test_host_prefill_rejects_small_workspace():
    x = make_prefill(1, 2, 128, 128, [256], torch.bfloat16, seed=80, packed=False)
    hx = _host(x)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdn.GDNError) as e:
        gdn.gdn_chunk_prefill_host(hx["q"], hx["k"], hx["v"], hx["g"], hx["beta"], workspace=ws,
                                   device="cuda")
    assert e.value.status == gdn.GDN_ERR_WORKSPACE
