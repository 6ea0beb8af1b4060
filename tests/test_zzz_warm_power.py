"""GPU parity of the warm-started power iteration (SIGNMUON_PI_WARM).

Each spectral scale's power iteration starts from the iterate the same problem
ended with in the previous step ([paper] "SignMuon: 通信高效的分布式Muon优化",
Algorithm 1's P power iterations, with the iterate carried across steps).

Power iteration composes: on a constant Gram matrix, t warm steps of P
iterations run exactly the arithmetic of one cold start with P*t iterations,
so the GPU's scales must match a cold handle bit for bit.  Against the
oracle, the warm-started estimates of each step are compared on the GPU's own
momentum.  The file name sorts it after the other GPU suites.
"""
import numpy as np
import pytest

import synth
from oracle import signmuon_ref as ref

from gpu_helpers import dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402

SHAPES = [(64, 96), (130, 70), (3, 5)]
SCALE_RTOL = {"bf16": 1e-2, "fp32": 1e-4}


def _handle(M, K, P, precision, flags=0, beta=0.0):
    f = flags | (smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0)
    return smo.SignMuon(SHAPES, M, beta=beta, lam=0.0, K=K, eps=1e-7, scale="spectral", P=P, flags=f)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("post_polar", [False, True])
def test_warm_steps_equal_a_cold_start_with_more_iterations(precision, post_polar):
    """beta = 0 and lambda = 0 with the same gradients every step keep the
    momentum, hence every Gram matrix, constant; K = 0 keeps the signs (so
    the post-vote majority) constant too.  After t warm steps with P = 1 the
    scales equal those of one step of a cold handle with P = t, bit for bit
    (the post-vote scales overwrite worker 0's row)."""
    M = 3
    extra = smo.SIGNMUON_POST_POLAR if post_polar else 0
    d = synth.numel(SHAPES)
    G = [dev(g) for g in synth.gradients(SHAPES, M, 1.0, step=1, config_id=81)]
    warm = _handle(M, 0, 1, precision, extra | smo.SIGNMUON_PI_WARM)
    W = torch.zeros(d, device="cuda")
    for t in range(1, 4):
        warm.step(W, G, 0.01)
        got = warm.get_scales()
        cold = _handle(M, 0, t, precision, extra)
        W2 = torch.zeros(d, device="cuda")
        cold.step(W2, G, 0.01)
        want = cold.get_scales()
        assert np.array_equal(got, want), f"step {t}: {got} vs {want}"
        cold.close()
    # the estimates do move between steps (the state is carried, not reset)
    first = _handle(M, 0, 1, precision, extra)
    first.step(torch.zeros(d, device="cuda"), G, 0.01)
    assert not np.array_equal(first.get_scales(), got)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_warm_scales_match_the_oracle_on_the_gpu_momentum(precision):
    """Fresh gradients every step (beta = 0.9): the oracle carries its own
    warm iterates over the GPU's momentum, step after step."""
    M, P, K = 2, 1, 5
    d = synth.numel(SHAPES)
    h = _handle(M, K, P, precision, smo.SIGNMUON_PI_WARM, beta=0.9)
    W = dev(synth.weights0(SHAPES, 83))
    state = [[None] * len(SHAPES) for _ in range(M)]
    for step in range(1, 4):
        G = synth.gradients(SHAPES, M, 1.0, step=step, config_id=83)
        h.step(W, [dev(g) for g in G], 0.01)
        got = h.get_scales()
        for m in range(M):
            t = torch.zeros(d, device="cuda")
            h.get_momentum(m, t)
            mom = host(t).astype(np.float64)
            for i, x in enumerate(ref.split(mom, SHAPES)):
                xw = x.T if x.shape[0] > x.shape[1] else x
                s, state[m][i] = ref.power_sigma(xw, P, state[m][i], return_u=True)
                rel = abs(float(got[m, i]) - s) / s
                assert rel <= SCALE_RTOL[precision], f"step {step} worker {m} matrix {i}: {rel:.3e}"


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_warm_state_restarts_after_a_zero_matrix(precision):
    """A zero momentum leaves a zero iterate; the next step starts cold, so
    it matches a fresh handle's first step bit for bit."""
    M = 2
    d = synth.numel(SHAPES)
    G = [dev(g) for g in synth.gradients(SHAPES, M, 1.0, step=1, config_id=85)]
    h = _handle(M, 3, 2, precision, smo.SIGNMUON_PI_WARM)
    W = torch.zeros(d, device="cuda")
    h.step(W, [torch.zeros(d, device="cuda") for _ in range(M)], 0.01)
    assert not h.get_scales().any()
    h.step(W, G, 0.01)
    cold = _handle(M, 3, 2, precision)
    cold.step(torch.zeros(d, device="cuda"), G, 0.01)
    assert np.array_equal(h.get_scales(), cold.get_scales())


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_warm_checkpoint_resume_bit_exact(precision):
    """A warm-started handle's checkpoint is W, the momentum and the
    power-iteration state (signmuon_get/set_pi_state): two steps, a save,
    and two more on a fresh handle equal four straight steps bit for bit;
    restoring only the momentum restarts the power iteration cold."""
    M, K, P, seed = 2, 3, 1, 87
    flags = smo.SIGNMUON_PI_WARM | smo.SIGNMUON_POST_POLAR
    d = synth.numel(SHAPES)

    def grads(step):
        return [dev(g) for g in synth.gradients(SHAPES, M, 1.0, step=step, config_id=seed)]

    straight = _handle(M, K, P, precision, flags, beta=0.9)
    Wa = dev(synth.weights0(SHAPES, seed))
    for step in range(1, 5):
        straight.step(Wa, grads(step), 0.01)

    first = _handle(M, K, P, precision, flags, beta=0.9)
    Wb = dev(synth.weights0(SHAPES, seed))
    for step in (1, 2):
        first.step(Wb, grads(step), 0.01)
    info = smo.signmuon_info(first.h)
    assert info["pi_state_workers"] == M * sum(min(r, c) for r, c in SHAPES)
    assert info["pi_state_single"] == sum(min(r, c) for r, c in SHAPES)
    mom = [torch.zeros(d, device="cuda") for _ in range(M)]
    for m in range(M):
        first.get_momentum(m, mom[m])
    s0 = torch.zeros(info["pi_state_workers"], device="cuda")
    s1 = torch.zeros(info["pi_state_single"], device="cuda")
    first.get_pi_state(0, s0)
    first.get_pi_state(1, s1)
    W_saved = Wb.clone()

    resumed = _handle(M, K, P, precision, flags, beta=0.9)
    cold = _handle(M, K, P, precision, flags, beta=0.9)
    W_cold = W_saved.clone()
    for m in range(M):
        resumed.set_momentum(m, mom[m])
        cold.set_momentum(m, mom[m])
    resumed.set_pi_state(0, s0)
    resumed.set_pi_state(1, s1)
    for step in (3, 4):
        resumed.step(W_saved, grads(step), 0.01)
        cold.step(W_cold, grads(step), 0.01)
    assert np.array_equal(host(W_saved).view(np.uint32), host(Wa).view(np.uint32))
    assert np.array_equal(resumed.get_scales(), straight.get_scales())
    assert not np.array_equal(cold.get_scales(), straight.get_scales())
    # a handle without the flag has no state to give
    plain = _handle(M, K, P, precision)
    with pytest.raises(smo.SignMuonError) as ei:
        plain.get_pi_state(0, s0)
    assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED
