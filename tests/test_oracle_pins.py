"""The CPU oracle against what the pages and mathematics fix (no GPU needed)."""

import pytest

import oracle_pins


@pytest.mark.parametrize("name", list(oracle_pins.ALL_PINS))
def test_pin(oracle, name):
    oracle_pins.ALL_PINS[name](oracle)


def test_state_size_equation_6():
    """Equation (6) of the SDM explainer (section 3.3): per-layer state
    (d_qk_total)^2 * d_v_total / (4 H^2) equals H * N * d_v for every workload,
    with d_qk_total = 2 sqrtN H and d_v_total = d_v H."""
    from sparse_memory_linear_pkm_b200 import synth

    for s in synth.WORKLOADS.values():
        d_qk_total = 2 * s.sqrt_n * s.H
        d_v_total = s.d_v * s.H
        assert d_qk_total ** 2 * d_v_total == 4 * s.H ** 2 * (s.H * s.N * s.d_v)


def test_isoflop_sizing():
    """isoFLOP sizing (SDM explainer section 3.2): d_qk_total = d/2 and
    d_v_total = d for the model width d each workload is derived from."""
    from sparse_memory_linear_pkm_b200 import synth

    widths = {"d2048_h16_n1024_dv128": 2048, "d2048_h4_n16384_dv512": 2048,
              "d4096_h8_n16384_dv512": 4096, "long_t1m_n262144_dv2048": 4096}
    for name, d in widths.items():
        s = synth.WORKLOADS[name]
        assert 2 * s.sqrt_n * s.H == d // 2 and s.d_v * s.H == d
        assert s.W == s.R == 64


def test_layer_forward_composes(oracle):
    """layer_forward = selection on k' and q', M0 broadcast over batch rows,
    then the recurrence."""
    import numpy as np

    rng = np.random.default_rng(3)
    B, T, H, sq, d_v, W, R = 2, 5, 2, 4, 3, 3, 2
    kp = rng.standard_normal((B, T, H, 2 * sq)).astype(np.float32)
    qp = rng.standard_normal((B, T, H, 2 * sq)).astype(np.float32)
    v = rng.standard_normal((B, T, H, d_v)).astype(np.float32)
    alpha = rng.random((B, T, H)).astype(np.float32)
    beta = rng.random((B, T, H)).astype(np.float32)
    M0 = rng.standard_normal((H, sq * sq, d_v)).astype(np.float32)
    out = oracle.layer_forward(kp, qp, v, alpha, beta, M0, W, R)
    iw, ww = oracle.pkm_topk(kp, W)
    ir, wr = oracle.pkm_topk(qp, R)
    y, M_T, _ = oracle.scan(iw, ww, ir, wr, v, alpha, beta, np.stack([M0] * B))
    assert np.array_equal(out["idx_w"], iw) and np.array_equal(out["idx_r"], ir)
    assert np.array_equal(out["y"], y) and np.array_equal(out["M_T"], M_T)
