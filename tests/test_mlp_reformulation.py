"""The two reformulations by which the TTT-MLP tensor-core kernel keeps its
products tensor-core shaped, checked in fp64 on random operands of the kernel's
shapes (b = 16 tokens, d = 64, hidden h = 256).  The dual form they rewrite is
the TTT write-up's (§03.7, extended to the MLP as §03.9 describes), which the
oracle pins separately; these identities are exact, so they hold to rounding."""
import numpy as np

B_, D, H = 16, 64, 256


def test_output_correction_after_the_update():
    """Zq2 W2 - tril(Zq2 X2^T) E3 = Zq2 W2' + striu(Zq2 X2^T) E3, W2' = W2 - X2^T E3:
    the kernel takes Zq3 from the updated W2 and adds the strictly-upper part."""
    rng = np.random.default_rng(0)
    Zq2, X2 = rng.standard_normal((B_, H)), rng.standard_normal((B_, H))
    W2, E3 = rng.standard_normal((H, D)), rng.standard_normal((B_, D))
    S2 = Zq2 @ X2.T
    lhs = Zq2 @ W2 - np.tril(S2) @ E3
    rhs = Zq2 @ (W2 - X2.T @ E3) + np.triu(S2, 1) @ E3
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(lhs) < 1e-13
    # The causal mask matters: with the full S2 the two sides differ.
    assert np.linalg.norm(lhs - (Zq2 @ (W2 - X2.T @ E3))) / np.linalg.norm(lhs) > 1e-3


def test_gram_over_hidden_blocks():
    """The [16 x 16] Gram Zq2 X2^T over the hidden width as one [64 x 64] product of
    rows (block, token): its four diagonal 16 x 16 blocks sum to the Gram."""
    rng = np.random.default_rng(1)
    Zq2, X2 = rng.standard_normal((B_, H)), rng.standard_normal((B_, H))
    nb = H // 64
    Zs = np.vstack([Zq2[:, 64 * g:64 * g + 64] for g in range(nb)])  # [(block, token), 64]
    Xs = np.vstack([X2[:, 64 * g:64 * g + 64] for g in range(nb)])
    R = Zs @ Xs.T
    gram = sum(R[B_ * g:B_ * g + B_, B_ * g:B_ * g + B_] for g in range(nb))
    ref = Zq2 @ X2.T
    assert np.linalg.norm(gram - ref) / np.linalg.norm(ref) < 1e-13
    # The off-diagonal blocks are cross terms that must not be added.
    wrong = sum(R[B_ * g:B_ * g + B_, B_ * ((g + 1) % nb):B_ * ((g + 1) % nb) + B_] for g in range(nb))
    assert np.linalg.norm(wrong - ref) / np.linalg.norm(ref) > 1e-1
