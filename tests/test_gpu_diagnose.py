"""The GPU residual-vs-full quantisation diagnostic against the oracle's: the same
synthetic loop sequence, reconstructions bit-exact (the codec and the chain are IEEE
operations with stated roundings), hence identical errors; and the diagnostic's claim
(residual error well below full at the same bit width) holds."""
import numpy as np
import pytest
import torch

from cross_loop_sparse_step_b200 import synth
from oracle import diagnostics as odiag

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,group", [(4, 32), (2, 64)])
def test_diagnostic_matches_oracle(bits, group):
    from cross_loop_sparse_step_b200 import diagnose
    K = synth.kv_loop_sequence(synth.rng(20 + bits), 1000, 4, 128, 4)
    want = odiag.residual_vs_full(K, bits, group)
    got = diagnose.residual_vs_full([torch.from_numpy(k).cuda() for k in K], bits, group)
    for r in range(1, 5):
        for kind in ("residual", "full"):
            a = got["hat_" + kind][r].cpu().numpy()
            assert np.array_equal(a.view(np.uint32), want["hat_" + kind][r].view(np.uint32)), (r, kind)
            assert abs(got[kind][r] - want[kind][r]) <= 1e-12 * want[kind][r]
        if r >= 2:
            assert got["residual"][r] < 0.5 * got["full"][r]
