"""A deferred error stays set until signmuon_sync reports it: with
SIGNMUON_ASYNC, a step whose momentum turns non-finite is followed by a
healthy step before the sync; the sync must still report E_NONFINITE, and
neither step may have moved W.  After the momentum is restored, steps update
W again.  The file name sorts it after the other GPU suites."""
import numpy as np
import pytest

import synth

from gpu_helpers import dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402


def test_deferred_error_survives_a_later_async_step():
    shapes = [(64, 96), (96, 64)]
    M, seed = 2, 53
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    bad = [g.copy() for g in G]
    bad[1][7] = np.inf
    h = smo.SignMuon(shapes, M, beta=0.9, lam=0.01, K=5, eps=1e-7, scale="spectral", P=2, flags=smo.SIGNMUON_ASYNC)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    W = dev(w0)
    h.step(W, [dev(g) for g in bad], 0.02)   # momentum turns non-finite: W must stay
    h.step(W, [dev(g) for g in G], 0.02)     # healthy gradients, but the error is unread
    with pytest.raises(smo.SignMuonError) as ei:
        h.sync()
    assert ei.value.status == smo.SIGNMUON_E_NONFINITE
    assert np.array_equal(host(W).view(np.uint32), w0.view(np.uint32))
    h.sync()                                  # cleared
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))       # restore the checkpointed momentum
    h.step(W, [dev(g) for g in G], 0.02)
    h.sync()
    # the same step on a fresh synchronous handle from the same state
    ref_h = smo.SignMuon(shapes, M, beta=0.9, lam=0.01, K=5, eps=1e-7, scale="spectral", P=2)
    for m in range(M):
        ref_h.set_momentum(m, dev(mom0[m]))
    W2 = dev(w0)
    ref_h.step(W2, [dev(g) for g in G], 0.02)
    assert np.array_equal(host(W).view(np.uint32), host(W2).view(np.uint32))
    assert not np.array_equal(host(W).view(np.uint32), w0.view(np.uint32))


def test_pipelined_host_steps_keep_w_after_a_deferred_error():
    """The same through signmuon_step_host with SIGNMUON_ASYNC, whose calls
    overlap (each call's gradients come in while the step before runs): the
    second of four queued calls has a non-finite gradient, so after one sync
    W_host holds the first call's update alone and the sync reports
    E_NONFINITE."""
    shapes = [(128, 256), (96, 160)]
    M, seed = 2, 59
    w0 = synth.weights0(shapes, seed)
    grads = [synth.gradients(shapes, M, 1.0, step=t, config_id=seed) for t in range(4)]
    grads[1][0][11] = np.nan
    h = smo.SignMuon(shapes, M, beta=0.9, lam=0.01, K=3, eps=1e-7, scale="fro", flags=smo.SIGNMUON_ASYNC)
    wt = torch.from_numpy(w0.copy()).pin_memory()
    gts = [[torch.from_numpy(g).pin_memory() for g in gs] for gs in grads]
    wh = wt.numpy()
    for t in range(4):
        h.step_host(wh, [g.numpy() for g in gts[t]], 0.02)
    with pytest.raises(smo.SignMuonError) as ei:
        h.sync()
    assert ei.value.status == smo.SIGNMUON_E_NONFINITE
    ref_h = smo.SignMuon(shapes, M, beta=0.9, lam=0.01, K=3, eps=1e-7, scale="fro")
    W2 = dev(w0)
    ref_h.step(W2, [dev(g) for g in grads[0]], 0.02)
    assert np.array_equal(wh.view(np.uint32), host(W2).view(np.uint32))
