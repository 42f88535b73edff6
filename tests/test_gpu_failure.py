"""Failure detection on the GPU without a fault: the bounded pipeline wait
gives up, reports GDLA_ERR_TIMEOUT through the status word, and the context
stays usable for the next forward pass."""
import pytest
import torch

import grouped_differential_attention_gdla_b200 as gdla
import oracle
from grouped_differential_attention_gdla_b200.inputs import custom, make_inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    from grouped_differential_attention_gdla_b200.build import build
    build()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdla.gdla_selftest_wait_timeout(status, 20_000_000)  # 20 ms on a barrier nothing completes
    torch.cuda.synchronize()
    assert int(status.item()) == gdla._binding.GDLA_ERR_TIMEOUT
    # the device is still healthy: a normal call succeeds and matches the oracle
    wl = custom(1, 200, 8, 2, 2, 64)
    x = {k: v.cuda() for k, v in make_inputs(wl, seed=3).items()}
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gdla.gdla_attn_fwd(x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"],
                             d_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    cpu = {k: v.cpu() for k, v in x.items()}
    ref = oracle.gdla_attn(cpu["q_sig"], cpu["q_noise"], cpu["k"], cpu["v"], cpu["lam"],
                           cpu["gate"])
    assert_parity(out.reshape(ref.shape).float().cpu().numpy(), ref, "after timeout")


def test_binding_status_word_checks():
    """The binding refuses a status word of the wrong dtype or device, and
    check_status() raises on a word a kernel has set, then clears it."""
    wl = custom(1, 64, 8, 2, 2, 64)
    x = {k: v.cuda() for k, v in make_inputs(wl, seed=4).items()}
    args = (x["q_sig"], x["q_noise"], x["k"], x["v"], x["lam"], x["gate"])
    with pytest.raises(ValueError):
        gdla.gdla_attn_fwd(*args, d_status=torch.zeros(1, dtype=torch.int16, device="cuda"))
    with pytest.raises(ValueError):
        gdla.gdla_attn_fwd(*args, d_status=torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError):
        gdla.gdla_attn_fwd(x["q_sig"], x["q_noise"].cpu(), *args[2:])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdla.gdla_selftest_wait_timeout(status, 1_000_000)
    with pytest.raises(gdla.GDLAError):
        gdla.check_status(d_status=status)
    gdla.check_status(d_status=status)  # cleared by the first check
    gdla.gdla_attn_fwd(*args)            # default status word
    gdla.check_status()
