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
