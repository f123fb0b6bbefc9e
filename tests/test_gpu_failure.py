"""Failure detection on the GPU without a fault: a bounded device wait that
nothing satisfies gives up, records MLA_ERR_TIMEOUT in the workspace error
word (the word every pipelined kernel of the library writes when a wait runs
out), and the same workspace then serves a clean call."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O  # noqa: E402


def test_bounded_wait_reports_timeout_and_workspace_recovers():
    from head_latent_attention_append_b200 import mla, workload
    s = workload.setup("tiny_fp32_decode", checked_count=1, check_all=True)
    mla.selftest_wait_timeout(s.ws, 1000)        # about 1 ms, then the wait gives up
    assert mla.get_error(s.ws) == -6             # MLA_ERR_TIMEOUT
    assert mla.status_string(-6) == "MLA_ERR_TIMEOUT"
    # The context is intact and the workspace is reusable: a decode through it
    # clears the word, reports nothing and matches the oracle.
    workload.step(s)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    wl = s.wl
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base)
    ref = O.mla_decode(dims, O.Weights(**s.host_weights.as_dict()), s.host_hidden[0], wl.n_q)
    got = s.out[0].cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-4 * np.abs(ref).max()


def test_timeout_is_reported_after_the_limit_not_before():
    """A 50 ms limit: the error word is set and the wait took at least that
    long on the device (CUDA events around the launch)."""
    from head_latent_attention_append_b200 import mla
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    mla.selftest_wait_timeout(ws, 50000)
    e1.record()
    torch.cuda.synchronize()
    assert mla.get_error(ws) == -6
    assert e0.elapsed_time(e1) >= 45.0
