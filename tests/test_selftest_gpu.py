"""Failure detection on the GPU without a fault: a launch whose bounded wait
cannot succeed gives up after its limit, the host reads TERN_ETIMEOUT once
from the device error word, and the next GEMV on the same context is still
bit-exact."""
import time

import numpy as np
import pytest

import oracle
from packed_ternary_weight_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ns", [1_000_000, 50_000_000])
def test_bounded_wait_expires_and_context_survives(limit_ns):
    assert torch.cuda.is_available()
    from packed_ternary_weight_b200 import tern
    assert tern.device_error() == tern.OK
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    tern.selftest_wait(limit_ns)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert limit_ns * 1e-9 <= dt < 5.0, dt
    assert tern.device_error() == tern.ETIMEOUT
    assert tern.device_error() == tern.OK            # read and cleared
    lay = synth.single_gemv_layer()
    d, buf = tern.pack_layer(lay)
    x = synth.draw_x_bf16(lay.seed, 1, lay.k)
    y = torch.empty(lay.n, dtype=torch.float32, device="cuda")
    tern.gemv(d, torch.from_numpy(buf).cuda(), tern.ACT_BF16_Q8, torch.from_numpy(x.view(np.int16)).cuda(), None,
              tern.OUT_F32, y)
    torch.cuda.synchronize()
    q, s = oracle.quantize_act(x)
    ref = oracle.gemv_bitnet_int8(lay.trits, q, s, lay.tensor_scale)[0]
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert tern.device_error() == tern.OK
