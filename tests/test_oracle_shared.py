"""Pins of the oracle's BF16 shared expert (DeepGEMM PR #416, BF16 shared-expert
test body): against an independent float64 numpy evaluation with torch's bf16
rounding between the steps, its SiTU form with and without the linear term,
a closed-form special case and token-permutation equivariance."""
import numpy as np
import pytest
import torch

import oracle


def bf16_bits(a) -> np.ndarray:
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_f64(b) -> np.ndarray:
    return oracle.bf16_bits_to_f32(b).astype(np.float64)


def draws(T, SH, SI, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn((T, SH), generator=g) * 0.25).to(torch.bfloat16)
    l1 = (torch.randn((2 * SI, SH), generator=g) * 0.02).to(torch.bfloat16)
    l2 = (torch.randn((SH, SI), generator=g) * 0.02).to(torch.bfloat16)
    u16 = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    return u16(x), u16(l1), u16(l2)


def reference(x, l1, l2, act):
    """float64 numpy products; torch rounds each step's result to bf16 (via fp32)."""
    SI = l1.shape[0] // 2
    gu = bits_f64(x) @ bits_f64(l1).T
    gu = bits_f64(bf16_bits(gu))
    g, u = gu[:, :SI], gu[:, SI:]
    h = bits_f64(bf16_bits(act(g, u)))
    return bf16_bits(h @ bits_f64(l2).T), bf16_bits(h)


def swiglu(g, u):
    return g / (1.0 + np.exp(-g)) * u


def situ(beta, lbeta):
    return lambda g, u: (1.0 / (1.0 + np.exp(-g))) * (beta * np.tanh(g / beta)) * (lbeta * np.tanh(u / lbeta))


def assert_close_bits(got, ref, what):
    """Equal bf16 bits but for rare one-ulp flips of values that sit on a
    rounding boundary (the sums run in different orders)."""
    d = np.abs(got.view(np.int16).astype(np.int32) - ref.view(np.int16).astype(np.int32))
    assert d.max() <= 1, (what, d.max())
    assert (d == 0).mean() >= 0.999, (what, (d == 0).mean())


@pytest.mark.parametrize("T,SH,SI,seed", [(5, 64, 32, 0), (3, 128, 96, 1), (7, 256, 128, 2)])
def test_shared_matches_float64_reference(T, SH, SI, seed):
    x, l1, l2 = draws(T, SH, SI, seed)
    got = oracle.shared_forward(x, l1, l2, intermediates=True)
    y_ref, h_ref = reference(x, l1, l2, swiglu)
    assert_close_bits(got["h"], h_ref, "h")
    assert_close_bits(got["y"], y_ref, "y")


def test_shared_situ_matches_float64_reference():
    x, l1, l2 = draws(4, 128, 64, 3)
    got = oracle.shared_forward(x, l1, l2, activation="situ", beta=1.25, linear_beta=1.5, intermediates=True)
    y_ref, h_ref = reference(x, l1, l2, situ(1.25, 1.5))
    assert_close_bits(got["h"], h_ref, "h")
    assert_close_bits(got["y"], y_ref, "y")


def test_shared_situ_without_linear_term_matches_float64_reference():
    """SiTU with no linear_beta: the up projection enters as it is,
    sigmoid(g) * beta * tanh(g / beta) * u (and differs from the form with a
    linear term)."""
    x, l1, l2 = draws(4, 128, 64, 8)
    got = oracle.shared_forward(x, l1, l2, activation="situ", beta=2.0, linear_beta=None, intermediates=True)
    plain = lambda g, u: (1.0 / (1.0 + np.exp(-g))) * (2.0 * np.tanh(g / 2.0)) * u
    y_ref, h_ref = reference(x, l1, l2, plain)
    assert_close_bits(got["h"], h_ref, "h")
    assert_close_bits(got["y"], y_ref, "y")
    clipped = oracle.shared_forward(x, l1, l2, activation="situ", beta=2.0, linear_beta=0.05)["y"]
    assert not np.array_equal(clipped, got["y"])


def test_shared_situ_with_large_betas_is_swiglu():
    """beta * tanh(g / beta) -> g and lbeta * tanh(u / lbeta) -> u as the betas
    grow, so SiTU with betas of 1e9 gives SwiGLU's bits."""
    x, l1, l2 = draws(5, 128, 64, 9)
    swig = oracle.shared_forward(x, l1, l2, intermediates=True)
    big = oracle.shared_forward(x, l1, l2, activation="situ", beta=1e9, linear_beta=1e9, intermediates=True)
    assert_close_bits(big["h"], swig["h"], "h")
    assert_close_bits(big["y"], swig["y"], "y")


def test_shared_gate_first_and_orientation():
    """Swapping the gate and up halves, or transposing L2's role, changes the
    result (the reference above takes gate = first SI rows of L1)."""
    x, l1, l2 = draws(4, 64, 64, 4)
    y = oracle.shared_forward(x, l1, l2)["y"]
    swapped = np.concatenate([l1[64:], l1[:64]])
    assert not np.array_equal(oracle.shared_forward(x, swapped, l2)["y"], y)
    assert not np.array_equal(oracle.shared_forward(x, l1, l2.T.copy())["y"], y)


def test_shared_closed_form_identity():
    """SH = SI = n, gate = 8 I, up = I, L2 = I: y = bf16(silu(8 x) * x) exactly
    per element (each dot product has a single nonzero term)."""
    n = 32
    rng = np.random.default_rng(5)
    xv = rng.uniform(-1, 1, (3, n)).astype(np.float32)
    x = bf16_bits(xv)
    eye = np.eye(n, dtype=np.float32)
    l1 = bf16_bits(np.concatenate([8 * eye, eye]))
    l2 = bf16_bits(eye)
    xd = bits_f64(x)
    g = bits_f64(bf16_bits(8 * xd))
    h = bits_f64(bf16_bits(g / (1.0 + np.exp(-g)) * xd))
    assert np.array_equal(oracle.shared_forward(x, l1, l2)["y"], bf16_bits(h))


def test_shared_token_permutation_equivariant():
    x, l1, l2 = draws(9, 128, 64, 6)
    y = oracle.shared_forward(x, l1, l2)["y"]
    perm = np.random.default_rng(7).permutation(9)
    assert np.array_equal(oracle.shared_forward(x, l1, l2, tokens=perm)["y"], y[perm])
    assert np.array_equal(oracle.shared_forward(x[perm], l1, l2)["y"], y[perm])
