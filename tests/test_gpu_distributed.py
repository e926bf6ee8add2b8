"""The building blocks of the sharded steps on the GPU, through the C ABI.

muon_step_direction must produce exactly the update direction (and momentum)
that muon_step applies, muon_apply must apply it exactly as muon_step does, and
the two sharded optimizers of muon_newton_schulz_04_b200.distributed, run with
their default CUDA functions on one rank, must match the fp64 oracle within the
step's tolerances (the whole-matrix one exchanges O in bf16, which adds at most
one bf16 rounding, 2^-8 relative, to the direction)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild
from muon_newton_schulz_04_b200.distributed import ShardedMuon, Zero1Muon

from parity import TOL_O, grad_tensor, make_groups

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    mbuild.build()


def _by_shape(w, *lists):
    return [tuple([lst[k] for k in idx] for lst in lists) for (_, _, idx) in w.groups()]


def test_step_direction_and_apply_reproduce_the_step():
    """On the GPT-2-small shapes (square, wide and tall matrices): the fp32 direction
    equals the O that muon_step applied and B is the same, bitwise; muon_apply with
    that O gives muon_step's weights bitwise; the bf16 direction is the fp32 one
    rounded to nearest."""
    w = wl.get(2)
    cfg = mb.config(weight_decay=0.1, scale_mode=mb.SCALE_MATCH_RMS, rms_target=0.2)
    G = [grad_tensor(g, w.grad_dtype) for g in wl.grads(w, 0)]
    W0 = [torch.from_numpy(x).cuda() for x in wl.weights(w)]
    # reference: muon_step, then its O
    ref = mb.Muon(cfg)
    W_ref = [x.clone() for x in W0]
    B_ref = [torch.zeros_like(x) for x in W0]
    ref.step(make_groups(w, W_ref, G, B_ref))
    idx = {k: (gi, j) for gi, (_, _, ks) in enumerate(w.groups()) for j, k in enumerate(ks)}
    O_ref = []
    for k in range(w.count):
        o = torch.empty_like(W0[k])
        ref.last_update(*idx[k], o)
        O_ref.append(o)
    torch.cuda.synchronize()
    # direction, then apply
    opt = mb.Muon(cfg)
    B = [torch.zeros_like(x) for x in W0]
    O32 = [torch.empty_like(x) for x in W0]
    opt.step_direction(_by_shape(w, G, B, O32))
    torch.cuda.synchronize()
    for k in range(w.count):
        assert torch.equal(O32[k], O_ref[k]), k
        assert torch.equal(B[k], B_ref[k]), k
    W = [x.clone() for x in W0]
    groups = [(Ws, Os, 1.0) for (Ws, Os) in _by_shape(w, W, O32)]
    opt.apply(groups)
    torch.cuda.synchronize()
    for k in range(w.count):
        assert torch.equal(W[k], W_ref[k]), k
    # bf16 direction from the same inputs (fresh momentum)
    B2 = [torch.zeros_like(x) for x in W0]
    O16 = [torch.empty(x.shape, dtype=torch.bfloat16, device="cuda") for x in W0]
    opt.step_direction(_by_shape(w, G, B2, O16))
    torch.cuda.synchronize()
    for k in range(w.count):
        assert torch.equal(O16[k], O_ref[k].to(torch.bfloat16)), k
    ref.close()
    opt.close()


def _check_against_oracle(w, W0, G, W, B_of, tol_o):
    for k in (0, 3, 4, 5, 40, 71):
        g64 = wl.widen(G[k], w.grad_dtype)
        res = oracle.muon_step(W0[k].astype(np.float64), g64, np.zeros(W0[k].shape), lr=0.02, momentum=0.95)
        Bk = B_of(k).double().cpu().numpy()
        assert np.max(np.abs(Bk - res["B"]) / np.maximum(np.abs(g64), 1e-30)) <= 1e-6, k
        err = np.linalg.norm(W[k].double().cpu().numpy() - res["W"])
        bound = 0.02 * tol_o * np.linalg.norm(res["O"]) + 1e-6 * np.linalg.norm(res["W"])
        assert err <= bound, (k, err, bound)


def test_sharded_muon_default_cuda_path_one_rank():
    w = wl.get(2)
    shapes = [(s.rows, s.cols) for s in w.matrices]
    opt = ShardedMuon(shapes, cfg=mb.config(), device=0)
    W0 = wl.weights(w)
    W = [torch.from_numpy(x).cuda() for x in W0]
    B = opt.new_momentum(W)
    G = wl.grads(w, 0)
    opt.step(W, [grad_tensor(g, w.grad_dtype) for g in G], B)
    torch.cuda.synchronize()
    assert opt.own == list(range(w.count))
    _check_against_oracle(w, W0, G, W, lambda k: B[k], TOL_O[mb.PREC_BF16] + 2.0 ** -8)


def test_zero1_muon_default_cuda_path_one_rank():
    w = wl.get(2)
    shapes = [(s.rows, s.cols) for s in w.matrices]
    opt = Zero1Muon(shapes, cfg=mb.config(), device=0)
    W0 = wl.weights(w)
    W = [torch.from_numpy(x).cuda() for x in W0]
    B = opt.new_momentum(W)
    G = wl.grads(w, 0)
    opt.step(W, [grad_tensor(g, w.grad_dtype) for g in G], B)
    torch.cuda.synchronize()
    _check_against_oracle(w, W0, G, W, lambda k: B[k], TOL_O[mb.PREC_BF16])


def test_direction_and_apply_reject_bad_arguments():
    """Checked before any launch: written buffers that overlap (O on B, W on O), a
    bad dtype code, and empty groups."""
    import ctypes
    L = mb.lib()
    opt = mb.Muon(mb.config())
    G = torch.randn(64, 32, device="cuda").to(torch.bfloat16)
    B = torch.zeros(64, 32, device="cuda")
    O = torch.empty(64, 32, device="cuda")
    W = torch.zeros(64, 32, device="cuda")
    with pytest.raises(mb.MuonError) as e:
        opt.step_direction([([G], [B], [B])])              # O is B
    assert e.value.status == mb.MUON_ERR_INVALID
    with pytest.raises(mb.MuonError) as e:
        opt.apply([([W], [W])])                            # W is O
    assert e.value.status == mb.MUON_ERR_INVALID
    pg = (ctypes.c_void_p * 1)(G.data_ptr())
    pb = (ctypes.c_void_p * 1)(B.data_ptr())
    po = (ctypes.c_void_p * 1)(O.data_ptr())
    grp = mb._DirGroup(64, 32, 1, mb.MUON_BF16, 7, ctypes.cast(pg, ctypes.POINTER(ctypes.c_void_p)),
                       ctypes.cast(pb, ctypes.POINTER(ctypes.c_void_p)), ctypes.cast(po, ctypes.POINTER(ctypes.c_void_p)))
    assert L.muon_step_direction(opt._h, ctypes.byref(grp), 1, None) == mb.MUON_ERR_INVALID
    assert L.muon_apply(opt._h, None, 0, None) == mb.MUON_ERR_INVALID
    assert torch.count_nonzero(B).item() == 0 and torch.count_nonzero(W).item() == 0
    opt.close()
