"""ctypes binding of libmuon_b200.so: argument marshalling only.

Every entry point of the C ABI (include/muon.h) is mirrored under the same
name.  Tensors are torch CUDA tensors; this module turns them into device
pointers and hands them to the library together with the current CUDA
stream.  No arithmetic of the optimizer happens here, and there is no
fallback: without the compiled library every call raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Iterable, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmuon_b200.so")

MUON_OK = 0
MUON_ERR_INVALID_ARG = 1
MUON_ERR_UNSUPPORTED = 2
MUON_ERR_WORKSPACE = 3
MUON_ERR_CUDA = 4
MUON_ERR_NONFINITE = 5
MUON_ERR_TIMEOUT = 6

MUON_F32 = 0
MUON_BF16 = 1

SCALE_MODES = {"original": 0, "match_rms_adamw": 1, "none": 2}

EXPORTED = [
    "muon_default_hparams", "muon_default_adamw_hparams", "muon_init", "muon_destroy",
    "muon_last_error", "muon_status_string", "muon_query_workspace", "muon_set_workspace",
    "muon_step", "muon_orthogonalize", "muon_adamw_step", "muon_newton_refresh",
    "muon_newton_precondition",
    "muon_check_device", "muon_selftest_wait", "muon_selftest_gemm", "muon_launch_count", "muon_profile_enable",
    "muon_profile_read",
    "muon_orthogonalize_noalloc", "muon_partition",
]

KERNEL_KINDS = ["momentum", "gram", "poly", "update", "apply", "adamw", "newton_refresh",
                "precondition", "other", "update_apply", "ns_small"]


class MuonError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


class Hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("momentum", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("eps", ctypes.c_float),
                ("ns_a", ctypes.c_float), ("ns_b", ctypes.c_float), ("ns_c", ctypes.c_float),
                ("nesterov", ctypes.c_int32), ("ns_steps", ctypes.c_int32),
                ("scale_mode", ctypes.c_int32), ("check_finite", ctypes.c_int32)]


class Group(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("count", ctypes.c_int32),
                ("grad_dtype", ctypes.c_int32), ("weights", ctypes.c_void_p),
                ("grads", ctypes.c_void_p), ("momentum", ctypes.c_void_p),
                ("update_out", ctypes.c_void_p), ("precond", ctypes.c_void_p),
                ("precond_blocks", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("precond_split", ctypes.c_void_p)]


class NsGroup(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("count", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("inputs", ctypes.c_void_p),
                ("outputs", ctypes.c_void_p)]


class AdamwTensor(ctypes.Structure):
    _fields_ = [("numel", ctypes.c_int64), ("grad_dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("param", ctypes.c_void_p),
                ("grad", ctypes.c_void_p), ("exp_avg", ctypes.c_void_p),
                ("exp_avg_sq", ctypes.c_void_p)]


class AdamwHparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float)]


class ActDesc(ctypes.Structure):
    _fields_ = [("acts", ctypes.c_void_p), ("act_dtype", ctypes.c_int32),
                ("nblocks", ctypes.c_int32), ("tokens", ctypes.c_int64),
                ("width", ctypes.c_int64), ("s_inv", ctypes.c_void_p),
                ("s_inv_split", ctypes.c_void_p)]


class KernelTimes(ctypes.Structure):
    _fields_ = [("ms", ctypes.c_double * len(KERNEL_KINDS)), ("launches", ctypes.c_uint64 * len(KERNEL_KINDS))]


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libmuon_b200.so (built in-tree).  Raises when it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m matrix_aware_optimizer_step_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    st = ctypes.c_int
    sig = {
        "muon_default_hparams": (None, [ctypes.POINTER(Hparams)]),
        "muon_default_adamw_hparams": (None, [ctypes.POINTER(AdamwHparams)]),
        "muon_init": (st, [ctypes.POINTER(vp), ctypes.c_int, sz]),
        "muon_destroy": (None, [vp]),
        "muon_last_error": (ctypes.c_char_p, [vp]),
        "muon_status_string": (ctypes.c_char_p, [st]),
        "muon_query_workspace": (st, [ctypes.POINTER(Group), i32, ctypes.POINTER(sz)]),
        "muon_set_workspace": (st, [vp, vp, sz]),
        "muon_step": (st, [vp, ctypes.POINTER(Group), i32, ctypes.POINTER(Hparams), vp]),
        "muon_orthogonalize": (st, [vp, ctypes.POINTER(NsGroup), i32, ctypes.POINTER(Hparams), vp]),
        "muon_adamw_step": (st, [vp, ctypes.POINTER(AdamwTensor), i32, ctypes.POINTER(AdamwHparams),
                                 i64, vp]),
        "muon_newton_refresh": (st, [vp, ctypes.POINTER(ActDesc), i32, ctypes.c_float, vp]),
        "muon_newton_precondition": (st, [vp, ctypes.POINTER(Group), i32, vp]),
        "muon_check_device": (st, [vp]),
        "muon_selftest_wait": (st, [vp, vp]),
        "muon_selftest_gemm": (st, [vp, vp]),
        "muon_launch_count": (ctypes.c_uint64, [vp]),
        "muon_profile_enable": (st, [vp, ctypes.c_int]),
        "muon_profile_read": (st, [vp, ctypes.POINTER(KernelTimes)]),
        "muon_orthogonalize_noalloc": (st, [vp, i32, i64, i64, vp, ctypes.POINTER(Hparams), vp]),
        "muon_partition": (st, [ctypes.POINTER(i64), ctypes.POINTER(i64), i32, i32,
                                ctypes.POINTER(i32)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def default_hparams(**over) -> Hparams:
    hp = Hparams()
    load_library().muon_default_hparams(ctypes.byref(hp))
    for k, v in over.items():
        if k == "scale_mode" and isinstance(v, str):
            v = SCALE_MODES[v]
        if k in ("nesterov", "check_finite"):
            v = int(bool(v))
        setattr(hp, k, v)
    return hp


def default_adamw_hparams(**over) -> AdamwHparams:
    hp = AdamwHparams()
    load_library().muon_default_adamw_hparams(ctypes.byref(hp))
    for k, v in over.items():
        setattr(hp, k, v)
    return hp


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def partition(shapes: Sequence, world: int) -> list:
    """Owner rank of every (rows, cols) matrix (muon_partition, host only)."""
    lib = load_library()
    n = len(shapes)
    rows = (ctypes.c_int64 * max(1, n))(*[int(s[0]) for s in shapes])
    cols = (ctypes.c_int64 * max(1, n))(*[int(s[1]) for s in shapes])
    own = (ctypes.c_int32 * max(1, n))()
    st = lib.muon_partition(rows, cols, n, int(world), own)
    if st != MUON_OK:
        raise MuonError(st, f"muon_partition: {lib.muon_status_string(st).decode()}")
    return [int(own[i]) for i in range(n)]


def orthogonalize_noalloc(x, out, hp: Optional[Hparams] = None, stream=None):
    """out (fp32) = Newton-Schulz of x, without a context and without any
    device allocation (the library's fixed scratch array is used)."""
    hp = hp or default_hparams()
    _check_cuda([x, out], "orthogonalize_noalloc")
    if tuple(out.shape) != tuple(x.shape) or x.dim() != 2:
        raise ValueError("x and out must be matrices of one shape")
    lib = load_library()
    st = lib.muon_orthogonalize_noalloc(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1],
                                        out.data_ptr(), ctypes.byref(hp), _stream_ptr(stream))
    if st != MUON_OK:
        raise MuonError(st, f"muon_orthogonalize_noalloc: {lib.muon_status_string(st).decode()}")


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return MUON_F32
    if t.dtype == torch.bfloat16:
        return MUON_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptrs(tensors: Sequence) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(1, len(tensors)))()
    for i, t in enumerate(tensors):
        arr[i] = t.data_ptr()
    return arr


def _check_cuda(ts: Iterable, what: str):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{what}: tensors must be contiguous CUDA tensors")


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class MuonContext:
    """One library context on one device (muon_init / muon_destroy)."""

    def __init__(self, device: int = 0, workspace_bytes: int = 0):
        self._lib = load_library()
        self._ctx = ctypes.c_void_p()
        self._ws = None
        st = self._lib.muon_init(ctypes.byref(self._ctx), int(device), int(workspace_bytes))
        if st != MUON_OK:
            raise MuonError(st, f"muon_init failed: {self._lib.muon_status_string(st).decode()}")
        self.device = device

    def close(self):
        if self._ctx:
            self._lib.muon_destroy(self._ctx)
            self._ctx = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _check(self, st: int, what: str):
        if st != MUON_OK:
            msg = self._lib.muon_last_error(self._ctx).decode()
            raise MuonError(st, f"{what}: {self._lib.muon_status_string(st).decode()}: {msg}")

    # -- groups ------------------------------------------------------------
    @staticmethod
    def make_groups(groups: Sequence[dict]):
        """Build muon_group structs from dicts with keys weights, grads,
        momentum (lists of tensors of one shape), optional update_out,
        precond (list of S^-1 tensors), precond_blocks and precond_split
        (the bf16 hi/lo splits a refresh wrote for those S^-1).  Returns the
        ctypes array and the objects that must stay alive during the call."""
        keep = []
        arr = (Group * max(1, len(groups)))()
        for i, g in enumerate(groups):
            grads = list(g["grads"])
            if not grads:
                raise ValueError("empty group")
            rows, cols = grads[0].shape
            for key in ("weights", "grads", "momentum", "update_out"):
                for t in (g.get(key) or []):
                    if tuple(t.shape) != (rows, cols):
                        raise ValueError(f"{key}: shape {tuple(t.shape)} != {(rows, cols)}")
            if g.get("precond") is not None:
                nb = int(g.get("precond_blocks", 1))
                d = cols // max(nb, 1)
                for t in g["precond"]:
                    if t.numel() != nb * d * d:
                        raise ValueError(f"precond: {t.numel()} elements != {nb} x {d} x {d}")
                for t in (g.get("precond_split") or []):
                    if t.numel() * t.element_size() != nb * 2 * d * d * 2:
                        raise ValueError(f"precond_split: {t.numel() * t.element_size()} bytes != "
                                         f"{nb} x 2 x {d} x {d} bf16")
            gs = arr[i]
            gs.rows, gs.cols, gs.count = rows, cols, len(grads)
            gs.grad_dtype = _dtype_code(grads[0])
            for key in ("weights", "grads", "momentum", "update_out", "precond", "precond_split"):
                ts = g.get(key)
                if ts is None:
                    setattr(gs, key, None)
                    continue
                ts = list(ts)
                _check_cuda(ts, key)
                p = _ptrs(ts)
                keep.append(p)
                setattr(gs, key, ctypes.cast(p, ctypes.c_void_p))
            gs.precond_blocks = int(g.get("precond_blocks", 1 if g.get("precond") is not None else 0))
        return arr, keep

    def query_workspace(self, groups: Sequence[dict]) -> int:
        arr, keep = self.make_groups(groups)
        n = ctypes.c_size_t()
        self._check(self._lib.muon_query_workspace(arr, len(groups), ctypes.byref(n)),
                    "muon_query_workspace")
        return n.value

    def set_workspace(self, tensor):
        """Use a caller-owned device buffer (e.g. a torch uint8 tensor) as
        workspace; None returns to library-owned workspace."""
        if tensor is None:
            self._check(self._lib.muon_set_workspace(self._ctx, None, 0), "muon_set_workspace")
            self._ws = None
            return
        self._check(self._lib.muon_set_workspace(self._ctx, tensor.data_ptr(),
                                                 tensor.numel() * tensor.element_size()),
                    "muon_set_workspace")
        self._ws = tensor

    def step(self, groups: Sequence[dict], hp: Optional[Hparams] = None, stream=None):
        hp = hp or default_hparams()
        groups = [g for g in groups if len(g["grads"]) > 0]
        arr, keep = self.make_groups(groups)
        self._check(self._lib.muon_step(self._ctx, arr, len(groups), ctypes.byref(hp),
                                        _stream_ptr(stream)), "muon_step")

    def orthogonalize(self, inputs: Sequence, outputs: Sequence, hp: Optional[Hparams] = None,
                      stream=None):
        """outputs[i] (fp32) = Newton-Schulz of inputs[i]; inputs grouped by
        shape and dtype automatically."""
        hp = hp or default_hparams()
        by = {}
        for x, o in zip(inputs, outputs):
            by.setdefault((tuple(x.shape), x.dtype), []).append((x, o))
        arr = (NsGroup * max(1, len(by)))()
        keep = []
        for i, ((shape, _), pairs) in enumerate(by.items()):
            xs = [p[0] for p in pairs]
            os_ = [p[1] for p in pairs]
            _check_cuda(xs + os_, "orthogonalize")
            pi, po = _ptrs(xs), _ptrs(os_)
            keep += [pi, po]
            arr[i].rows, arr[i].cols, arr[i].count = shape[0], shape[1], len(xs)
            arr[i].in_dtype = _dtype_code(xs[0])
            arr[i].inputs = ctypes.cast(pi, ctypes.c_void_p)
            arr[i].outputs = ctypes.cast(po, ctypes.c_void_p)
        self._check(self._lib.muon_orthogonalize(self._ctx, arr, len(by), ctypes.byref(hp),
                                                 _stream_ptr(stream)), "muon_orthogonalize")

    def adamw_step(self, params: Sequence, grads: Sequence, exp_avgs: Sequence,
                   exp_avg_sqs: Sequence, step: int, hp: Optional[AdamwHparams] = None,
                   stream=None):
        hp = hp or default_adamw_hparams()
        n = len(params)
        arr = (AdamwTensor * max(1, n))()
        for i in range(n):
            _check_cuda([params[i], grads[i], exp_avgs[i], exp_avg_sqs[i]], "adamw")
            arr[i].numel = params[i].numel()
            arr[i].grad_dtype = _dtype_code(grads[i])
            arr[i].param = params[i].data_ptr()
            arr[i].grad = grads[i].data_ptr()
            arr[i].exp_avg = exp_avgs[i].data_ptr()
            arr[i].exp_avg_sq = exp_avg_sqs[i].data_ptr()
        self._check(self._lib.muon_adamw_step(self._ctx, arr, n, ctypes.byref(hp), int(step),
                                              _stream_ptr(stream)), "muon_adamw_step")

    def newton_refresh(self, acts: Sequence, s_invs: Sequence, nblocks: Sequence[int],
                       damping: float = 0.0, stream=None, splits: Optional[Sequence] = None):
        """s_invs[i] (fp32, nblocks[i] x d x d) = inverse second moments of
        the column blocks of acts[i] (bf16 or fp32 tokens x width).  With
        splits, splits[i] (bf16, nblocks[i] x 2d x d, or None) also receives
        their hi/lo split, to pass to step() as a group's precond_split."""
        n = len(acts)
        arr = (ActDesc * max(1, n))()
        for i in range(n):
            _check_cuda([acts[i], s_invs[i]], "newton_refresh")
            arr[i].acts = acts[i].data_ptr()
            arr[i].act_dtype = _dtype_code(acts[i])
            arr[i].nblocks = int(nblocks[i])
            arr[i].tokens, arr[i].width = acts[i].shape
            arr[i].s_inv = s_invs[i].data_ptr()
            sp = splits[i] if splits is not None else None
            if sp is not None:
                _check_cuda([sp], "newton_refresh")
                d = arr[i].width // max(1, arr[i].nblocks)
                if sp.numel() * sp.element_size() != arr[i].nblocks * 2 * d * d * 2:
                    raise ValueError("newton_refresh: split buffer size")
                arr[i].s_inv_split = sp.data_ptr()
        self._check(self._lib.muon_newton_refresh(self._ctx, arr, n, float(damping),
                                                  _stream_ptr(stream)), "muon_newton_refresh")

    def newton_precondition(self, grads: Sequence, s_invs: Sequence, nblocks: int, outputs: Sequence,
                            stream=None):
        """outputs[i] (fp32) = grads[i] (bf16 rows x cols) right-multiplied
        block-diagonally by s_invs[i] (fp32, nblocks x d x d, d = cols /
        nblocks).  All grads share one shape."""
        grads = list(grads)
        if not grads:
            return
        arr, keep = self.make_groups([{"grads": grads, "update_out": list(outputs),
                                       "precond": list(s_invs), "precond_blocks": int(nblocks)}])
        self._check(self._lib.muon_newton_precondition(self._ctx, arr, 1, _stream_ptr(stream)),
                    "muon_newton_precondition")

    def check_device(self):
        self._check(self._lib.muon_check_device(self._ctx), "muon_check_device")

    def selftest_wait(self, stream=None):
        """Enqueue the failure-detection self test: a bounded device-side
        wait that runs out (2 s); check_device() then raises MUON_ERR_TIMEOUT."""
        self._check(self._lib.muon_selftest_wait(self._ctx, _stream_ptr(stream)), "muon_selftest_wait")

    def selftest_gemm(self, stream=None):
        """Enqueue the engine's failure-detection self test: a Gram launch
        whose MMA thread never issues, so its producer, MMA thread and
        epilogue waits all run out (2 s) and abort; check_device() then
        raises MUON_ERR_TIMEOUT."""
        self._check(self._lib.muon_selftest_gemm(self._ctx, _stream_ptr(stream)), "muon_selftest_gemm")

    @property
    def launch_count(self) -> int:
        return int(self._lib.muon_launch_count(self._ctx))

    def profile(self, enable: bool):
        self._check(self._lib.muon_profile_enable(self._ctx, int(bool(enable))), "muon_profile_enable")

    def profile_read(self) -> dict:
        """{kind: (total ms, launches)} since the last read (synchronises)."""
        kt = KernelTimes()
        self._check(self._lib.muon_profile_read(self._ctx, ctypes.byref(kt)), "muon_profile_read")
        return {k: (kt.ms[i], int(kt.launches[i])) for i, k in enumerate(KERNEL_KINDS)}
