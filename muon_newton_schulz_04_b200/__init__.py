"""Python binding of the B200 Muon step library (include/muon.h).

Argument marshalling only: torch tensors are turned into raw pointers, sizes
and the current CUDA stream, and every entry point of the C ABI is called by
the same name.  All arithmetic runs in the CUDA kernels of libmuon_b200.so;
there is no fallback.  If the shared library is missing, the first call raises.

    import torch, muon_newton_schulz_04_b200 as mb
    opt = mb.Muon(mb.config(lr=0.02, weight_decay=0.1))
    opt.step([mb.Group(W=[w1, w2], G=[g1, g2], B=[b1, b2])])   # same-shape matrices per group
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import List, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmuon_b200.so")

MUON_OK, MUON_ERR_INVALID, MUON_ERR_UNSUPPORTED, MUON_ERR_OOM, MUON_ERR_CUDA, MUON_ERR_DEVICE_TIMEOUT = range(6)
MUON_BF16, MUON_FP32 = 0, 1
PREC_BF16, PREC_FP32_DEBUG = 0, 1
SCALE_NONE, SCALE_MATCH_RMS, SCALE_CUSTOM = 0, 1, 2
NS_GRAM, NS_POLY, NS_UPDATE = 0, 1, 2


class MuonConfig(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("momentum", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("eps", ctypes.c_float), ("rms_target", ctypes.c_float), ("nesterov", ctypes.c_int),
                ("ns_steps", ctypes.c_int), ("ns_a", ctypes.c_float), ("ns_b", ctypes.c_float),
                ("ns_c", ctypes.c_float), ("scale_mode", ctypes.c_int), ("precision", ctypes.c_int)]


class _Group(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("count", ctypes.c_int),
                ("grad_dtype", ctypes.c_int), ("scale", ctypes.c_float),
                ("W", ctypes.POINTER(ctypes.c_void_p)), ("G", ctypes.POINTER(ctypes.c_void_p)),
                ("B", ctypes.POINTER(ctypes.c_void_p))]


class _OrthoGroup(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("count", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("M", ctypes.POINTER(ctypes.c_void_p)),
                ("O", ctypes.POINTER(ctypes.c_void_p))]


class _DirGroup(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("count", ctypes.c_int),
                ("grad_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("G", ctypes.POINTER(ctypes.c_void_p)), ("B", ctypes.POINTER(ctypes.c_void_p)),
                ("O", ctypes.POINTER(ctypes.c_void_p))]


class _ApplyGroup(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("count", ctypes.c_int),
                ("o_dtype", ctypes.c_int), ("scale", ctypes.c_float),
                ("W", ctypes.POINTER(ctypes.c_void_p)), ("O", ctypes.POINTER(ctypes.c_void_p))]


class _PhaseArgs(ctypes.Structure):
    _fields_ = [("phase", ctypes.c_int), ("precision", ctypes.c_int), ("m", ctypes.c_int), ("n", ctypes.c_int),
                ("count", ctypes.c_int), ("alpha", ctypes.c_float), ("beta", ctypes.c_float),
                ("x_op", ctypes.c_void_p), ("a_in", ctypes.c_void_p), ("x_master", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("out_op", ctypes.c_void_p)]


_LIB: Optional[ctypes.CDLL] = None

# name -> (restype, argtypes)
_SIGNATURES = {
    "muon_config_default": (None, [ctypes.POINTER(MuonConfig)]),
    "muon_validate_config": (ctypes.c_int, [ctypes.POINTER(MuonConfig)]),
    "muon_validate_groups": (ctypes.c_int, [ctypes.POINTER(_Group), ctypes.c_int]),
    "muon_create": (ctypes.c_int, [ctypes.POINTER(MuonConfig), ctypes.c_int, ctypes.POINTER(ctypes.c_void_p)]),
    "muon_set_config": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(MuonConfig)]),
    "muon_set_memory_limit": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t]),
    "muon_memory_held": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_size_t)]),
    "muon_step": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(_Group), ctypes.c_int, ctypes.c_void_p]),
    "muon_step_host": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(_Group), ctypes.c_int, ctypes.c_void_p]),
    "muon_step_direction": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(_DirGroup), ctypes.c_int, ctypes.c_void_p]),
    "muon_apply": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(_ApplyGroup), ctypes.c_int, ctypes.c_void_p]),
    "muon_orthogonalize": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(_OrthoGroup), ctypes.c_int, ctypes.c_void_p]),
    "muon_ns_phase_run": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(_PhaseArgs), ctypes.c_void_p]),
    "muon_qk_clip": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_void_p]),
    "muon_sync": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "muon_last_norms": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_float), ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]),
    "muon_last_update_rms": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_float), ctypes.c_int,
                                            ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]),
    "muon_last_update": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "muon_timing_enable": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int]),
    "muon_timing_read": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int),
                                        ctypes.c_int, ctypes.c_void_p]),
    "muon_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "muon_last_error": (ctypes.c_char_p, [ctypes.c_void_p]),
    "muon_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "muon_momentum_norm_noalloc": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int,
                                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_char_p, ctypes.c_int]),
    "muon_plan_units": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int)]),
    "muon_plan_tile_m": (ctypes.c_int, []),
    "muon_plan_tile_n": (ctypes.c_int, []),
    "muon_plan_tiles": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]),
}


def lib() -> ctypes.CDLL:
    """The loaded C library.  Raises if libmuon_b200.so has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m muon_newton_schulz_04_b200.build` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


class MuonError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{lib().muon_status_string(status).decode()}: {msg}")
        self.status = status


def config(**kw) -> MuonConfig:
    """Default configuration (lr 0.02, momentum 0.95 Nesterov, 5 steps, (3.4445, -4.775, 2.0315), eps 1e-7)
    with the given fields replaced."""
    c = MuonConfig()
    lib().muon_config_default(ctypes.byref(c))
    for k, v in kw.items():
        if k not in dict(MuonConfig._fields_):
            raise TypeError(f"unknown config field {k}")
        setattr(c, k, int(v) if isinstance(getattr(c, k), int) else float(v))
    return c


@dataclasses.dataclass
class Group:
    """Same-shape matrices: W (fp32, updated), G (bf16 or fp32), B (fp32 momentum, updated)."""
    W: Sequence
    G: Sequence
    B: Sequence
    scale: float = 1.0


def _ptrs(ts) -> "ctypes.Array":
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = t.data_ptr()
    return arr


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return MUON_BF16
    if t.dtype == torch.float32:
        return MUON_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check_tensors(ts, shape, on_cuda: bool, dtype=None, device: Optional[int] = None):
    """Same shape, dense, on the expected device kind and, when given, of one dtype
    (the library reads and writes these buffers as dense arrays of that type) and on
    CUDA device `device` (the kernels run on one device and take only its memory)."""
    for t in ts:
        if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
            raise ValueError(f"expected contiguous tensors of shape {tuple(shape)}, got {tuple(t.shape)}")
        if t.is_cuda != on_cuda:
            raise ValueError("tensor on the wrong device kind")
        if on_cuda and device is not None and t.device.index != device:
            raise ValueError(f"tensor on cuda:{t.device.index}, expected cuda:{device}")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"expected {dtype} tensors, got {t.dtype}")


def _stream(stream, device: Optional[int] = None) -> int:
    """The raw cudaStream_t: the given stream, else the current stream of `device`
    (of the current device when None)."""
    import torch
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


class Muon:
    """A handle of the C library bound to one CUDA device."""

    def __init__(self, cfg: Optional[MuonConfig] = None, device: int = 0):
        self._h = ctypes.c_void_p()
        self.cfg = cfg if cfg is not None else config()
        st = lib().muon_create(ctypes.byref(self.cfg), int(device), ctypes.byref(self._h))
        if st != MUON_OK:
            raise MuonError(st, f"muon_create on device {device}")
        self.device = device
        self._keep = []

    # ------------------------------------------------------------------ helpers
    def _check(self, st: int, what: str):
        if st != MUON_OK:
            raise MuonError(st, f"{what}: {lib().muon_last_error(self._h).decode()}")

    def _groups(self, groups: List[Group], on_cuda: bool):
        arr = (_Group * len(groups))()
        keep = []
        for i, g in enumerate(groups):
            import torch
            rows, cols = g.W[0].shape
            _check_tensors(g.W, (rows, cols), on_cuda, torch.float32, self.device)
            _check_tensors(g.G, (rows, cols), on_cuda, g.G[0].dtype, self.device)
            _check_tensors(g.B, (rows, cols), on_cuda, torch.float32, self.device)
            if not (len(g.W) == len(g.G) == len(g.B)):
                raise ValueError("W, G and B lists differ in length")
            pw, pg, pb = _ptrs(g.W), _ptrs(g.G), _ptrs(g.B)
            keep += [pw, pg, pb]
            arr[i] = _Group(rows, cols, len(g.W), _dtype_code(g.G[0]), float(g.scale),
                            ctypes.cast(pw, ctypes.POINTER(ctypes.c_void_p)),
                            ctypes.cast(pg, ctypes.POINTER(ctypes.c_void_p)),
                            ctypes.cast(pb, ctypes.POINTER(ctypes.c_void_p)))
        return arr, keep

    # ------------------------------------------------------------------ API
    def set_config(self, cfg: MuonConfig):
        self._check(lib().muon_set_config(self._h, ctypes.byref(cfg)), "muon_set_config")
        self.cfg = cfg

    def set_memory_limit(self, nbytes: int):
        """Caps the device bytes the handle may hold (0: no cap); a call that would grow
        past it raises MuonError (MUON_ERR_OOM) before launching anything."""
        self._check(lib().muon_set_memory_limit(self._h, int(nbytes)), "muon_set_memory_limit")

    def memory_held(self) -> int:
        n = ctypes.c_size_t(0)
        self._check(lib().muon_memory_held(self._h, ctypes.byref(n)), "muon_memory_held")
        return n.value

    def step(self, groups: List[Group], stream=None):
        arr, keep = self._groups(groups, True)
        self._shapes = [(arr[i].rows, arr[i].cols, arr[i].count) for i in range(len(groups))]
        self._check(lib().muon_step(self._h, arr, len(groups), ctypes.c_void_p(_stream(stream, self.device))), "muon_step")

    def step_host(self, groups: List[Group], stream=None):
        arr, keep = self._groups(groups, False)
        self._shapes = [(arr[i].rows, arr[i].cols, arr[i].count) for i in range(len(groups))]
        self._check(lib().muon_step_host(self._h, arr, len(groups), ctypes.c_void_p(_stream(stream, self.device))), "muon_step_host")

    def step_direction(self, groups, stream=None):
        """groups: list of (G_list, B_list, O_list) of same-shape matrices.  B is updated
        and O (fp32 or bf16 tensors of W's shape) receives the Newton-Schulz direction;
        no weight is touched (see muon_step_direction)."""
        import torch
        arr = (_DirGroup * len(groups))()
        keep = []
        for i, (Gs, Bs, Os) in enumerate(groups):
            rows, cols = Bs[0].shape
            if not (len(Gs) == len(Bs) == len(Os)):
                raise ValueError("G, B and O lists differ in length")
            _check_tensors(Gs, (rows, cols), True, Gs[0].dtype, self.device)
            _check_tensors(Bs, (rows, cols), True, torch.float32, self.device)
            _check_tensors(Os, (rows, cols), True, Os[0].dtype, self.device)
            pg, pb, po = _ptrs(Gs), _ptrs(Bs), _ptrs(Os)
            keep += [pg, pb, po]
            arr[i] = _DirGroup(rows, cols, len(Bs), _dtype_code(Gs[0]), _dtype_code(Os[0]),
                               ctypes.cast(pg, ctypes.POINTER(ctypes.c_void_p)),
                               ctypes.cast(pb, ctypes.POINTER(ctypes.c_void_p)),
                               ctypes.cast(po, ctypes.POINTER(ctypes.c_void_p)))
        self._check(lib().muon_step_direction(self._h, arr, len(groups), ctypes.c_void_p(_stream(stream, self.device))),
                    "muon_step_direction")

    def apply(self, groups, stream=None):
        """groups: list of (W_list, O_list[, scale]) of same-shape matrices:
        W <- W - lr*wd*W - lr*s*O (see muon_apply); O fp32 or bf16."""
        import torch
        arr = (_ApplyGroup * len(groups))()
        keep = []
        for i, grp in enumerate(groups):
            Ws, Os = grp[0], grp[1]
            scale = float(grp[2]) if len(grp) > 2 else 1.0
            rows, cols = Ws[0].shape
            if len(Ws) != len(Os):
                raise ValueError("W and O lists differ in length")
            _check_tensors(Ws, (rows, cols), True, torch.float32, self.device)
            _check_tensors(Os, (rows, cols), True, Os[0].dtype, self.device)
            pw, po = _ptrs(Ws), _ptrs(Os)
            keep += [pw, po]
            arr[i] = _ApplyGroup(rows, cols, len(Ws), _dtype_code(Os[0]), scale,
                                 ctypes.cast(pw, ctypes.POINTER(ctypes.c_void_p)),
                                 ctypes.cast(po, ctypes.POINTER(ctypes.c_void_p)))
        self._check(lib().muon_apply(self._h, arr, len(groups), ctypes.c_void_p(_stream(stream, self.device))),
                    "muon_apply")

    def orthogonalize(self, groups, stream=None):
        """groups: list of (M_list, O_list); O = NS(M / (||M||_F + eps)), fp32 outputs."""
        arr = (_OrthoGroup * len(groups))()
        keep = []
        for i, (Ms, Os) in enumerate(groups):
            import torch
            rows, cols = Ms[0].shape
            _check_tensors(Ms, (rows, cols), True, Ms[0].dtype, self.device)
            _check_tensors(Os, (rows, cols), True, torch.float32, self.device)
            pm, po = _ptrs(Ms), _ptrs(Os)
            keep += [pm, po]
            arr[i] = _OrthoGroup(rows, cols, len(Ms), _dtype_code(Ms[0]),
                                 ctypes.cast(pm, ctypes.POINTER(ctypes.c_void_p)),
                                 ctypes.cast(po, ctypes.POINTER(ctypes.c_void_p)))
        self._check(lib().muon_orthogonalize(self._h, arr, len(groups), ctypes.c_void_p(_stream(stream, self.device))),
                    "muon_orthogonalize")

    def ns_phase(self, phase: int, precision: int, m: int, n: int, count: int, alpha: float, beta: float,
                 x_op=None, a_in=None, x_master=None, out=None, out_op=None, stream=None):
        for t in (x_op, a_in, x_master, out, out_op):
            if t is not None and (not t.is_cuda or t.device.index != self.device):
                raise ValueError(f"building-block buffers must be on cuda:{self.device}")
        p = lambda t: None if t is None else t.data_ptr()
        args = _PhaseArgs(phase, precision, m, n, count, alpha, beta, p(x_op), p(a_in), p(x_master), p(out), p(out_op))
        self._check(lib().muon_ns_phase_run(self._h, ctypes.byref(args), ctypes.c_void_p(_stream(stream, self.device))),
                    "muon_ns_phase_run")

    def qk_clip(self, Wq, Wk, max_logits, head_dim: int, tau: float, stream=None):
        """MuonClip's QK-Clip: rows of head h of Wq and Wk times sqrt(min(1, tau / max_logits[h]))."""
        import torch
        for name, t in (("Wq", Wq), ("Wk", Wk), ("max_logits", max_logits)):
            if t is None and name == "Wk":
                continue
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
            if t.device.index != self.device:
                raise ValueError(f"{name} is on cuda:{t.device.index}, the handle on cuda:{self.device}")
        n_heads = max_logits.numel()
        if Wq.dim() != 2:
            raise ValueError("Wq must be 2-D")
        rows, cols = Wq.shape
        if rows != n_heads * head_dim or (Wk is not None and tuple(Wk.shape) != (rows, cols)):
            raise ValueError("Wq / Wk must be (n_heads * head_dim) x cols")
        self._check(lib().muon_qk_clip(self._h, ctypes.c_void_p(Wq.data_ptr()),
                                       None if Wk is None else ctypes.c_void_p(Wk.data_ptr()),
                                       ctypes.c_void_p(max_logits.data_ptr()), n_heads, head_dim, cols, float(tau),
                                       ctypes.c_void_p(_stream(stream, self.device))), "muon_qk_clip")

    def sync(self, stream=None):
        self._check(lib().muon_sync(self._h, ctypes.c_void_p(_stream(stream, self.device))), "muon_sync")

    def last_norms(self, stream=None) -> List[float]:
        n = ctypes.c_int(0)
        lib().muon_last_norms(self._h, None, 0, ctypes.byref(n), ctypes.c_void_p(_stream(stream, self.device)))
        buf = (ctypes.c_float * max(n.value, 1))()
        self._check(lib().muon_last_norms(self._h, buf, n.value, ctypes.byref(n), ctypes.c_void_p(_stream(stream, self.device))),
                    "muon_last_norms")
        return list(buf[: n.value])

    def last_update_rms(self, stream=None) -> List[float]:
        """Per matrix (groups in order), the RMS of the update lr * s * O of the last step."""
        n = ctypes.c_int(0)
        lib().muon_last_update_rms(self._h, None, 0, ctypes.byref(n), ctypes.c_void_p(_stream(stream, self.device)))
        buf = (ctypes.c_float * max(n.value, 1))()
        self._check(lib().muon_last_update_rms(self._h, buf, n.value, ctypes.byref(n),
                                               ctypes.c_void_p(_stream(stream, self.device))), "muon_last_update_rms")
        return list(buf[: n.value])

    def last_update(self, group: int, index: int, dst, stream=None):
        """O of matrix `index` of group `group` of the last step, written to dst (fp32,
        the matrix's rows x cols, contiguous, on the device)."""
        import torch
        shapes = getattr(self, "_shapes", None)
        if shapes is None or not (0 <= group < len(shapes)) or not (0 <= index < shapes[group][2]):
            raise ValueError(f"no matrix {index} in group {group} of the last call")
        _check_tensors([dst], shapes[group][:2], True, torch.float32, self.device)
        self._check(lib().muon_last_update(self._h, group, index, ctypes.c_void_p(dst.data_ptr()),
                                           ctypes.c_void_p(_stream(stream, self.device))), "muon_last_update")

    TIMING_KINDS = ("momentum_norm", "norm_finalize", "gram", "poly", "update", "apply")

    def timing(self, enable: bool = True):
        self._check(lib().muon_timing_enable(self._h, int(enable)), "muon_timing_enable")

    def timing_read(self, stream=None):
        """{phase: (total ms, launches)} since the last read (synchronises the stream)."""
        k = len(self.TIMING_KINDS)
        ms = (ctypes.c_double * k)()
        n = (ctypes.c_int * k)()
        self._check(lib().muon_timing_read(self._h, ms, n, k, ctypes.c_void_p(_stream(stream, self.device))), "muon_timing_read")
        return {name: (ms[i], n[i]) for i, name in enumerate(self.TIMING_KINDS)}

    def close(self):
        if self._h:
            lib().muon_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def momentum_norm_noalloc(G, B, norm_out, U_out=None, momentum: float = 0.95, nesterov: bool = True, stream=None):
    """Momentum phase of one matrix with no device allocation (see muon.h):
    B <- momentum*B + G in place, U_out = G + momentum*B (or B), norm_out[0] = ||U||_F."""
    import torch
    rows, cols = B.shape
    if not B.is_cuda:
        raise ValueError("B must be a CUDA tensor")
    dev = B.device.index
    _check_tensors([G], (rows, cols), True, None, dev)
    _check_tensors([B], (rows, cols), True, torch.float32, dev)
    if U_out is not None:
        _check_tensors([U_out], (rows, cols), True, torch.float32, dev)
    if norm_out.dtype != torch.float32 or not norm_out.is_cuda or norm_out.numel() < 1:
        raise ValueError("norm_out must be a float32 CUDA tensor with at least one element")
    if norm_out.device.index != dev:
        raise ValueError(f"norm_out is on cuda:{norm_out.device.index}, B on cuda:{dev}")
    err = ctypes.create_string_buffer(256)
    # the entry point works on the current device: make it B's for the call
    with torch.cuda.device(dev):
        st = lib().muon_momentum_norm_noalloc(rows, cols, _dtype_code(G), G.data_ptr(), B.data_ptr(),
                                              None if U_out is None else U_out.data_ptr(), float(momentum),
                                              int(nesterov), norm_out.data_ptr(), ctypes.c_void_p(_stream(stream)),
                                              err, 256)
    if st != MUON_OK:
        raise MuonError(st, f"muon_momentum_norm_noalloc: {err.value.decode()}")


def plan_tiles(shapes, phase: int):
    """Tile list of a grouped GEMM launch: [(group, matrix, tile_row, tile_col)] (host only)."""
    flat = (ctypes.c_int * (3 * len(shapes)))(*[int(v) for s in shapes for v in s])
    n = ctypes.c_int(0)
    lib().muon_plan_tiles(flat, len(shapes), phase, None, 0, ctypes.byref(n))
    out = (ctypes.c_int * (4 * max(n.value, 1)))()
    st = lib().muon_plan_tiles(flat, len(shapes), phase, out, n.value, ctypes.byref(n))
    if st != MUON_OK:
        raise MuonError(st, "muon_plan_tiles")
    return [tuple(out[4 * i: 4 * i + 4]) for i in range(n.value)]


def plan_units(shapes, phase: int, clusters: int, split: bool = False):
    """Work units of a two-CTA GEMM launch (host only): tuples (cluster, group, matrix,
    tile_row, tile_col, k_begin, k_end, kind, slot, nslots, n_half)."""
    flat = (ctypes.c_int * (3 * len(shapes)))(*[int(v) for s in shapes for v in s])
    n = ctypes.c_int(0)
    lib().muon_plan_units(flat, len(shapes), phase, clusters, int(split), None, 0, ctypes.byref(n))
    out = (ctypes.c_int * (11 * max(n.value, 1)))()
    st = lib().muon_plan_units(flat, len(shapes), phase, clusters, int(split), out, n.value, ctypes.byref(n))
    if st != MUON_OK:
        raise MuonError(st, "muon_plan_units")
    return [tuple(out[11 * i: 11 * i + 11]) for i in range(n.value)]


def tile_shape():
    return lib().muon_plan_tile_m(), lib().muon_plan_tile_n()
