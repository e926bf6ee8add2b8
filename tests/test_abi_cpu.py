"""The C-ABI library on the host: it builds, loads, exports every declared symbol,
validates arguments without a GPU, and plans tile lists that cover every output
element exactly once."""
import ctypes
import json
import os
import re

import numpy as np
import pytest
import torch

import muon_newton_schulz_04_b200 as mb
from muon_newton_schulz_04_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session", autouse=True)
def built_library():
    mbuild.build()
    return mb.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "muon.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?(muon_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 18
    L = ctypes.CDLL(mb.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(mb._SIGNATURES), set(names) ^ set(mb._SIGNATURES)


def test_library_links_no_cuda_driver_at_load_time():
    out = os.popen(f"ldd {mb.LIB_PATH}").read()
    assert "libcuda.so" not in out
    assert "libcudart" not in out          # runtime linked statically


def test_default_config_matches_printed_coefficients():
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "ns_coefficients.json")))
    c = mb.config()
    assert (c.ns_a, c.ns_b, c.ns_c) == tuple(np.float32(v) for v in (g["a"], g["b"], g["c"]))
    assert c.ns_steps == g["steps"] and c.nesterov == 1
    assert abs(c.momentum - 0.95) < 1e-7 and abs(c.lr - 0.02) < 1e-9 and abs(c.eps - 1e-7) < 1e-13
    assert mb.lib().muon_validate_config(ctypes.byref(c)) == mb.MUON_OK


@pytest.mark.parametrize("field,value", [("momentum", 1.0), ("momentum", -0.1), ("ns_steps", -1), ("ns_steps", 17),
                                         ("nesterov", 2), ("lr", float("nan")), ("weight_decay", -1.0),
                                         ("eps", float("inf")), ("scale_mode", 7), ("precision", 3),
                                         ("ns_a", float("inf"))])
def test_config_validation_rejects(field, value):
    c = mb.config()
    setattr(c, field, value)
    assert mb.lib().muon_validate_config(ctypes.byref(c)) == mb.MUON_ERR_INVALID


def test_match_rms_needs_positive_target():
    c = mb.config(scale_mode=mb.SCALE_MATCH_RMS, rms_target=0.0)
    assert mb.lib().muon_validate_config(ctypes.byref(c)) == mb.MUON_ERR_INVALID
    c = mb.config(scale_mode=mb.SCALE_MATCH_RMS, rms_target=0.2)
    assert mb.lib().muon_validate_config(ctypes.byref(c)) == mb.MUON_OK


def _group(rows=4, cols=8, count=2, dtype=mb.MUON_BF16, ptr=0x10000, w=None, g=None, b=None):
    arrs = []
    def mk(vals):
        a = (ctypes.c_void_p * count)(*vals)
        arrs.append(a)
        return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))
    W = mk(w if w is not None else [ptr + 0x1000 * k for k in range(count)])
    G = mk(g if g is not None else [ptr + 0x100000 + 0x1000 * k for k in range(count)])
    B = mk(b if b is not None else [ptr + 0x200000 + 0x1000 * k for k in range(count)])
    grp = mb._Group(rows, cols, count, dtype, 1.0, W, G, B)
    return grp, arrs


def test_group_validation():
    L = mb.lib()
    g, keep = _group()
    assert L.muon_validate_groups(ctypes.byref(g), 1) == mb.MUON_OK
    assert L.muon_validate_groups(None, 1) == mb.MUON_ERR_INVALID
    assert L.muon_validate_groups(ctypes.byref(g), 0) == mb.MUON_ERR_INVALID
    for kw in [dict(rows=0), dict(cols=-3), dict(count=0), dict(dtype=5),
               dict(w=[0x10000, 0]), dict(b=[0x10000, 0x10002]), dict(g=[0x10001, 0x20000])]:
        g2, keep2 = _group(**kw)
        assert L.muon_validate_groups(ctypes.byref(g2), 1) == mb.MUON_ERR_INVALID, kw
    g3, keep3 = _group(rows=1 << 16, cols=1 << 16)          # 2^32 elements
    assert L.muon_validate_groups(ctypes.byref(g3), 1) == mb.MUON_ERR_INVALID
    g4, keep4 = _group(dtype=mb.MUON_FP32, g=[0x10002, 0x20000])   # fp32 needs 4-byte alignment
    assert L.muon_validate_groups(ctypes.byref(g4), 1) == mb.MUON_ERR_INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_create_without_gpu_reports_cuda_error():
    h = ctypes.c_void_p()
    c = mb.config()
    st = mb.lib().muon_create(ctypes.byref(c), 0, ctypes.byref(h))
    assert st in (mb.MUON_ERR_CUDA, mb.MUON_ERR_INVALID)
    assert not h.value
    assert mb.lib().muon_step(None, None, 0, None) == mb.MUON_ERR_INVALID
    assert mb.lib().muon_destroy(None) == mb.MUON_ERR_INVALID
    assert mb.lib().muon_set_memory_limit(None, 1 << 20) == mb.MUON_ERR_INVALID
    held = ctypes.c_size_t(7)
    assert mb.lib().muon_memory_held(None, ctypes.byref(held)) == mb.MUON_ERR_INVALID
    assert held.value == 7


def test_status_strings():
    L = mb.lib()
    assert L.muon_status_string(mb.MUON_OK) == b"MUON_OK"
    assert L.muon_status_string(mb.MUON_ERR_DEVICE_TIMEOUT) == b"MUON_ERR_DEVICE_TIMEOUT"


# ----------------------------------------------------------------------------- planner

def _coverage(shapes, phase):
    BM, BN = mb.tile_shape()
    tiles = mb.plan_tiles(shapes, phase)
    dims = [(min(r, c), max(r, c), k) for (r, c, k) in shapes]
    cover = {}
    for g, (m, n, k) in enumerate(dims):
        cols = n if phase == 2 else m
        cover[g] = np.zeros((k, m, cols), dtype=np.int32)
    costs = []
    for (g, z, ti, tj) in tiles:
        m, n, k = dims[g]
        costs.append(n if phase == 0 else m)
        r0, c0 = ti * BM, tj * BN
        rows = np.arange(r0, min(r0 + BM, m))
        if phase == 2:
            cols = np.arange(c0, min(c0 + BN, n))
            cover[g][z][np.ix_(rows, cols)] += 1
            continue
        cols = np.arange(c0, min(c0 + BN, m))
        R, C = np.meshgrid(rows, cols, indexing="ij")
        direct = C >= R                      # the epilogue's store masks
        mirror = C > R
        np.add.at(cover[g][z], (R[direct], C[direct]), 1)
        np.add.at(cover[g][z], (C[mirror], R[mirror]), 1)
    return cover, costs


@pytest.mark.parametrize("shapes", [[(256, 512, 1)], [(4096, 4096, 1)], [(768, 768, 4), (3072, 768, 1), (768, 3072, 1)],
                                    [(1600, 1600, 2), (6400, 1600, 1)], [(37, 1000, 1), (1000, 37, 2)], [(1, 64, 1), (64, 1, 1)],
                                    [(2048, 1408, 2), (16384, 4096, 1)]])
@pytest.mark.parametrize("phase", [0, 1, 2])
def test_tiles_cover_every_output_exactly_once(shapes, phase):
    cover, costs = _coverage(shapes, phase)
    for g, c in cover.items():
        assert c.min() == 1 and c.max() == 1, (g, c.min(), c.max())
    assert costs == sorted(costs, reverse=True)        # longest tiles first


def test_symmetric_tiles_skip_the_lower_triangle():
    BM, BN = mb.tile_shape()
    full = len(mb.plan_tiles([(4096, 4096, 1)], 2))
    sym = len(mb.plan_tiles([(4096, 4096, 1)], 0))
    assert full == (4096 // BM) * (4096 // BN)
    assert sym < 0.56 * full


UNIT_CASES = [([(4096, 4096, 1)], 74), ([(4096, 4096, 1)], 5), ([(256, 512, 1)], 74),
              ([(768, 768, 4), (3072, 768, 1)], 74), ([(2048, 1408, 3)], 74),
              ([(1024, 1536, 1)], 74), ([(1600, 1600, 2), (6400, 1600, 1)], 74)]


def _kblocks(shapes, phase, tiles):
    dims = [(min(r, c), max(r, c)) for (r, c, _) in shapes]
    return {t: ((dims[t[0]][1] if phase == 0 else dims[t[0]][0]) + 63) // 64 for t in tiles}


@pytest.mark.parametrize("shapes,clusters", UNIT_CASES)
@pytest.mark.parametrize("phase", [0, 1, 2])
def test_split_units_cover_each_k_block_once_and_never_chain_waits(shapes, clusters, phase):
    units = mb.plan_units(shapes, phase, clusters, split=True)
    tiles = mb.plan_tiles(shapes, phase)
    kbl = _kblocks(shapes, phase, tiles)
    seen = {t: [] for t in tiles}
    by_cluster = {}
    slots = {}
    for (c, g, z, tr, tc, kb, ke, kind, slot, nsl, nh) in units:
        assert nh == 0
        seen[(g, z, tr, tc)].append((kb, ke, kind, slot, nsl, c))
        by_cluster.setdefault(c, []).append(kind)
        if kind == 2:
            assert slot not in slots
            slots[slot] = (g, z, tr, tc, kb)
    for t, parts in seen.items():
        parts.sort()
        assert parts, t
        cover = [(kb, ke) for (kb, ke, *_r) in parts]
        assert cover[0][0] == 0 and cover[-1][1] == kbl[t]
        assert all(cover[i][1] == cover[i + 1][0] for i in range(len(cover) - 1))     # contiguous, no overlap
        if len(parts) == 1:
            assert parts[0][2] == 0
        else:
            head = parts[0]
            assert head[2] == 1 and head[4] == len(parts) - 1
            for i, p in enumerate(parts[1:]):
                assert p[2] == 2 and p[3] == head[3] + i                            # slots in K order
                assert p[5] != head[5]                                              # another cluster
    for c, kinds in by_cluster.items():
        # a waiting head is its cluster's last unit and each cluster produces at most one
        # partial, before any wait: producers never wait, so waits cannot chain
        assert all(k != 1 for k in kinds[:-1]) and kinds.count(2) <= 1
    assert set(c for (c, *_r) in units) <= set(range(clusters))


@pytest.mark.parametrize("shapes,clusters", UNIT_CASES)
@pytest.mark.parametrize("phase", [0, 1, 2])
def test_default_units_cover_each_tile_once(shapes, clusters, phase):
    units = mb.plan_units(shapes, phase, clusters, split=False)
    tiles = mb.plan_tiles(shapes, phase)
    kbl = _kblocks(shapes, phase, tiles)
    seen = {t: [] for t in tiles}
    load = {}
    for (c, g, z, tr, tc, kb, ke, kind, slot, nsl, nh) in units:
        assert kind == 0 and kb == 0 and ke == kbl[(g, z, tr, tc)]
        seen[(g, z, tr, tc)].append((nh, c))
        load[c] = load.get(c, 0) + (1.0 if nh == 0 else 0.5)
    for t, parts in seen.items():
        halves = sorted(nh for (nh, _c) in parts)
        assert halves in ([0], [1, 2]), (t, parts)
        if halves == [1, 2]:
            assert parts[0][1] != parts[1][1]                                       # halves on two clusters
    T = len(tiles)
    assert max(load.values()) <= -(-T // clusters)                                  # never worse than whole tiles
    if T >= clusters and 0 < 2 * (T % clusters) <= clusters:
        assert max(load.values()) == T // clusters + 0.5                            # the tail round is halved


def test_no_undefined_library_symbols():
    out = os.popen(f"nm -D --undefined-only {mb.LIB_PATH}").read()
    assert "muon" not in out


def test_group_validation_rejects_overlapping_written_buffers():
    """W and B are updated in place: they may not share memory with any W, G or B of
    the call.  Gradients are only read and may be shared."""
    L = mb.lib()
    ok_cases = [dict(w=[0x10000, 0x10080]),                     # 4 x 8 fp32 = 128 B: adjacent is fine
                dict(g=[0x300000, 0x300000]),                   # one gradient read by both matrices
                dict(g=[0x300000, 0x300020])]                   # bf16 gradients overlapping each other
    for kw in ok_cases:
        g, keep = _group(**kw)
        assert L.muon_validate_groups(ctypes.byref(g), 1) == mb.MUON_OK, kw
    bad_cases = [dict(w=[0x10000, 0x10000]),                    # the same W twice
                 dict(w=[0x10000, 0x10040]),                    # partial overlap of two W
                 dict(b=[0x10000, 0x211000]),                   # B[0] is W[0]
                 dict(g=[0x10000, 0x300000]),                   # G[0] is W[0]
                 dict(g=[0x210040, 0x300000])]                  # G[0] inside B[0] (at 0x210000)
    for kw in bad_cases:
        g, keep = _group(**kw)
        assert L.muon_validate_groups(ctypes.byref(g), 1) == mb.MUON_ERR_INVALID, kw
    # across groups: the second group's W is the first group's B[1] (at 0x211000)
    g1, k1 = _group()
    g2, k2 = _group(count=1, w=[0x211000], g=[0x500000], b=[0x600000])
    arr = (mb._Group * 2)(g1, g2)
    assert L.muon_validate_groups(arr, 2) == mb.MUON_ERR_INVALID
    g2b, k2b = _group(count=1, w=[0x700000], g=[0x500000], b=[0x600000])
    arr = (mb._Group * 2)(g1, g2b)
    assert L.muon_validate_groups(arr, 2) == mb.MUON_OK


def test_qk_clip_binding_checks_tensors_before_the_library():
    """The binding refuses tensors the fp32 kernel cannot read safely (wrong dtype,
    device or layout, or a head count that does not match the rows) before any call
    into the library."""
    import torch
    opt = mb.Muon.__new__(mb.Muon)               # no device handle: nothing may reach the library
    opt._h = ctypes.c_void_p()
    opt.device = 0
    Wq = torch.zeros(8, 4)
    S = torch.ones(2)
    with pytest.raises(ValueError):
        opt.qk_clip(Wq, None, S, 4, 10.0)                          # CPU tensors
    with pytest.raises(ValueError):
        opt.qk_clip(Wq.to(torch.bfloat16), None, S, 4, 10.0)       # not float32
    with pytest.raises(ValueError):
        opt.qk_clip(torch.zeros(4, 8).t(), None, S, 4, 10.0)       # not contiguous


def test_binding_checks_buffer_dtypes_before_the_library():
    """W and B are read and written as fp32 and the gradients of a group share one
    dtype; last_update needs an fp32 buffer of the matrix's shape.  The binding
    refuses anything else before any call into the library."""
    import torch
    opt = mb.Muon.__new__(mb.Muon)
    opt._h = ctypes.c_void_p()
    opt.device = 0
    W, B = torch.zeros(4, 8), torch.zeros(4, 8)
    G = torch.zeros(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        opt.step_host([mb.Group(W=[W.to(torch.bfloat16)], G=[G], B=[B])])
    with pytest.raises(ValueError):
        opt.step_host([mb.Group(W=[W], G=[G], B=[B.double()])])
    with pytest.raises(ValueError):
        opt.step_host([mb.Group(W=[W, W.clone()], G=[G, G.float()], B=[B, B.clone()])])
    with pytest.raises(ValueError):
        opt.last_update(0, 0, torch.zeros(4, 8))              # no call has recorded any matrix


class _FakeCudaTensor:
    """Stands in for a CUDA tensor on a machine without a GPU: just the attributes
    the binding inspects before it calls the library."""

    def __init__(self, shape, dtype, index):
        self.shape, self.dtype, self.is_cuda = tuple(shape), dtype, True
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True

    def data_ptr(self):
        raise AssertionError("a wrong-device tensor reached the library call")

    def numel(self):
        return int(np.prod(self.shape))


def test_binding_refuses_tensors_of_another_device():
    """The kernels of a handle run on its device and take only that device's memory:
    a W, G, B, output or building-block buffer on another GPU is refused by the
    binding before any call into the library.  The no-allocation call takes its
    device from B and refuses the other buffers when they live elsewhere."""
    opt = mb.Muon.__new__(mb.Muon)
    opt._h = ctypes.c_void_p()
    opt.device = 0
    f32, bf = torch.float32, torch.bfloat16
    on0 = lambda dt=f32: _FakeCudaTensor((4, 8), dt, 0)
    on1 = lambda dt=f32: _FakeCudaTensor((4, 8), dt, 1)
    for W, G, B in ((on1(), on0(bf), on0()), (on0(), on1(bf), on0()), (on0(), on0(bf), on1())):
        with pytest.raises(ValueError, match="cuda:1"):
            opt.step([mb.Group(W=[W], G=[G], B=[B])])
    with pytest.raises(ValueError, match="cuda:1"):
        opt.orthogonalize([([on0()], [on1()])])
    with pytest.raises(ValueError, match="cuda:0"):
        opt.ns_phase(mb.NS_GRAM, mb.PREC_BF16, 8, 8, 1, 1.0, 0.0, x_op=on1(bf), out=on0(bf))
    opt._shapes = [(4, 8, 1)]
    with pytest.raises(ValueError, match="cuda:1"):
        opt.last_update(0, 0, on1())
    n1 = _FakeCudaTensor((1,), f32, 1)
    with pytest.raises(ValueError, match="cuda:1"):
        mb.momentum_norm_noalloc(on1(bf), on0(), _FakeCudaTensor((1,), f32, 0))
    with pytest.raises(ValueError, match="cuda:1"):
        mb.momentum_norm_noalloc(on0(bf), on0(), n1)
    with pytest.raises(ValueError, match="cuda:1"):
        mb.momentum_norm_noalloc(on0(bf), on0(), _FakeCudaTensor((1,), f32, 0), U_out=on1())


def test_direction_and_apply_reject_a_null_handle():
    """The two entry points of the sharded step refuse a NULL handle on the host
    (their other argument checks run on a handle and are tested on the GPU)."""
    L = mb.lib()
    assert L.muon_step_direction(None, None, 0, None) == mb.MUON_ERR_INVALID
    assert L.muon_apply(None, None, 0, None) == mb.MUON_ERR_INVALID
