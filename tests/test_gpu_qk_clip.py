"""QK-Clip kernel against the oracle: per-element parity and the capped logits."""
import numpy as np
import pytest
import torch

import oracle
import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("heads,hd,cols", [(12, 64, 768), (25, 64, 1600), (3, 5, 7)])
def test_qk_clip_matches_oracle(heads, hd, cols):
    mbuild.build()
    rng = np.random.default_rng(heads * hd + cols)
    Wq = rng.standard_normal((heads * hd, cols)).astype(np.float32)
    Wk = rng.standard_normal((heads * hd, cols)).astype(np.float32)
    S = rng.uniform(10, 300, size=heads).astype(np.float32)
    tau = 100.0
    opt = mb.Muon(mb.config())
    dq, dk, dS = torch.from_numpy(Wq).cuda(), torch.from_numpy(Wk).cuda(), torch.from_numpy(S).cuda()
    opt.qk_clip(dq, dk, dS, hd, tau)
    opt.sync()
    rq, rk = oracle.qk_clip(Wq.astype(np.float64), Wk.astype(np.float64), S.astype(np.float64), tau, hd)
    for got, ref, orig in ((dq, rq, Wq), (dk, rk, Wk)):
        g = got.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(g - ref) / (np.abs(ref) + 1e-30)) <= 1e-6
        for h in range(heads):                   # heads under tau: untouched bits
            if S[h] <= tau:
                assert np.array_equal(got.cpu().numpy()[h * hd:(h + 1) * hd], orig[h * hd:(h + 1) * hd])
    with pytest.raises(mb.MuonError):
        opt.qk_clip(dq, dk, dS, hd, -1.0)
    opt.close()
