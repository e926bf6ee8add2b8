"""The no-allocation entry point against the regular step.

muon_momentum_norm_noalloc serves callers that cannot allocate device memory
(a runtime with its own fixed device pool, code running while another component
holds the allocator): it updates the momentum buffer and reports ||U||_F using
only a static scratch array.  Here it must give the same momentum buffer and the
same norms as muon_step / muon_last_norms on the same inputs, on two calls in a
row, within the momentum tolerance of the other tests (1e-6 relative).  This file
is named to be collected last."""
import numpy as np
import pytest
import torch

import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,dtype", [(768, 3072, torch.bfloat16), (1000, 37, torch.float32),
                                             (4096, 4096, torch.bfloat16)])
def test_noalloc_momentum_matches_step_on_two_calls(rows, cols, dtype):
    mbuild.build()
    torch.cuda.set_device(0)
    rng = np.random.default_rng(rows + cols)
    Gs = [torch.from_numpy(rng.standard_normal((rows, cols)).astype(np.float32)).to(dtype).cuda() for _ in range(2)]
    mu = 0.95
    # regular path: muon_step on a scratch weight, then the last norms
    opt = mb.Muon(mb.config(momentum=mu, nesterov=1))
    W = torch.zeros(rows, cols, device="cuda")
    B_ref = torch.zeros(rows, cols, device="cuda")
    # no-allocation path
    B_na = torch.zeros(rows, cols, device="cuda")
    U_na = torch.empty(rows, cols, device="cuda")
    norm_na = torch.empty(1, device="cuda")
    for G in Gs:
        B_old = B_ref.clone()
        opt.step([mb.Group(W=[W], G=[G], B=[B_ref])])
        ref_norm = opt.last_norms()[0]
        mb.momentum_norm_noalloc(G, B_na, norm_na, U_out=U_na, momentum=mu, nesterov=True)
        torch.cuda.synchronize()
        den = (mu * B_old.abs() + G.float().abs()).clamp_min(1e-30)
        assert float(((B_na - B_ref).abs() / den).max()) <= 1e-6
        assert abs(float(norm_na[0]) - ref_norm) <= 1e-6 * ref_norm
        U_ref = G.double() + mu * B_ref.double()
        assert float(((U_na.double() - U_ref).abs() / (den.double() * (1 + mu))).max()) <= 1e-6
    opt.close()


def test_noalloc_rejects_oversize_and_bad_arguments():
    mbuild.build()
    G = torch.zeros(8, 8, device="cuda")
    B = torch.zeros(8, 8, device="cuda")
    n = torch.empty(1, device="cuda")
    with pytest.raises(mb.MuonError) as e:
        mb.momentum_norm_noalloc(G, B, n, momentum=1.5)
    assert e.value.status == mb.MUON_ERR_INVALID
    L = mb.lib()
    rows = cols = 1 << 15                       # 2^30 elements > 2^29 limit
    err = __import__("ctypes").create_string_buffer(256)
    st = L.muon_momentum_norm_noalloc(rows, cols, mb.MUON_FP32, G.data_ptr(), B.data_ptr(), None, 0.9, 1,
                                      n.data_ptr(), None, err, 256)
    assert st == mb.MUON_ERR_UNSUPPORTED and b"no-allocation limit" in err.value
    # written buffers may not overlap: U_out is B, U_out inside G, norm inside B
    for u, nrm in ((B, n), (G, n), (None, B[0, :1])):
        with pytest.raises(mb.MuonError) as e:
            mb.momentum_norm_noalloc(G, B, nrm, U_out=u)
        assert e.value.status == mb.MUON_ERR_INVALID
    st = L.muon_momentum_norm_noalloc(8, 8, mb.MUON_FP32, G.data_ptr(), G.data_ptr() + 16, None, 0.9, 1,
                                      n.data_ptr(), None, err, 256)
    assert st == mb.MUON_ERR_INVALID and b"overlap" in err.value


def test_noalloc_calls_leave_free_device_memory_unchanged():
    """After one warm-up call (which may load the module and place the static array),
    further calls take no device memory: the free bytes the driver reports stay the
    same across calls, and torch's allocator holds no more than before."""
    mbuild.build()
    torch.cuda.set_device(0)
    rows, cols = 2048, 1536
    G = torch.randn(rows, cols, device="cuda").to(torch.bfloat16)
    B = torch.zeros(rows, cols, device="cuda")
    U = torch.empty(rows, cols, device="cuda")
    n = torch.empty(1, device="cuda")
    mb.momentum_norm_noalloc(G, B, n, U_out=U)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    held0 = torch.cuda.memory_reserved()
    for _ in range(5):
        mb.momentum_norm_noalloc(G, B, n, U_out=U)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_reserved() == held0
