"""The failure path on the GPU, without a fault: a bounded device-side wait that nothing satisfies gives
up after its limit, the kernel records HCSA_ERR_TIMEOUT in the device status word and returns; the host
reads (and clears) the status, and the context keeps working for the next call."""
import time

import numpy as np
import pytest
import torch

import synth
from tests._helpers import dev

pytestmark = pytest.mark.gpu

HCSA_ERR_TIMEOUT = 7


def test_bounded_wait_reports_timeout_and_context_survives():
    import long_context_compressed_05_b200 as h
    from long_context_compressed_05_b200 import PrefillLayer
    assert h.hcsa_get_device_status() == 0
    t0 = time.time()
    h.hcsa_selftest_wait_timeout()
    status = h.hcsa_get_device_status()
    assert status == HCSA_ERR_TIMEOUT
    assert time.time() - t0 < 60            # the wait gave up on its own
    assert h.hcsa_get_device_status() == 0  # the read cleared the word
    # the context still runs a layer end to end
    spec = synth.LayerSpec(kind="csa", T=300, D=256, m=4, width=8, C=256, di=64, Hi=8, topk=64, window=128, H=8,
                           dh=128, scale=128 ** -0.5, dtype="bf16", seed=91)
    inp = synth.prefill_inputs(spec)
    layer = PrefillLayer(spec)
    out = layer.forward(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]))
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == 0
    assert torch.isfinite(out.float()).all()
    assert np.abs(out.float().cpu().numpy()).max() > 0


HCSA_ERR_DEVICE = 9


@pytest.mark.parametrize("H,dh,C", [(8, 128, 256), (64, 512, 1024)])   # generic and tensor-core attention
def test_selection_outside_the_visible_range_is_skipped_and_reported(H, dh, C):
    """A caller-provided selection index that is neither -1 padding nor a visible entry (here: one entry
    past the visible range, and one far beyond the sequence) is not read: the kernel checks the index
    before the access, skips that key, and records HCSA_ERR_DEVICE.  The output equals the one computed
    with those indices replaced by -1."""
    import long_context_compressed_05_b200 as h
    from long_context_compressed_05_b200 import PrefillLayer
    spec = synth.LayerSpec(kind="csa", T=900, D=256, m=4, width=8, C=C, di=64, Hi=8, topk=128, window=128, H=H,
                           dh=dh, scale=dh ** -0.5, dtype="bf16", seed=92)
    inp = synth.prefill_inputs(spec)
    layer = PrefillLayer(spec)
    layer.forward(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]))
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == 0
    t = 801                                          # 200 visible entries, 128 selected
    bad = layer.sel.clone()
    bad[t, 5] = t // spec.m                          # first entry that is not yet visible
    bad[t, 9] = 1 << 30                              # far beyond the sequence
    good = bad.clone()
    good[t, 5] = -1
    good[t, 9] = -1
    layer.attend(sel=good)
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == 0
    want = layer.out.clone()
    layer.attend(sel=bad)
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == HCSA_ERR_DEVICE
    assert h.hcsa_get_device_status() == 0
    assert torch.equal(layer.out, want)
