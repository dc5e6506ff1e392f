"""ctypes binding of libfipa.so (include/fipa.h).  Argument marshalling only.

Every step of the forward runs in the CUDA library; this module checks
shapes/dtypes of torch tensors, allocates outputs and the workspace with torch,
and passes raw device pointers and the current CUDA stream.  There is no
fallback: if the library is missing or the call fails, it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfipa.so")

FIPA_OK = 0
STATUS_NAMES = {0: "FIPA_OK", 1: "FIPA_ERR_INVALID_ARG", 2: "FIPA_ERR_UNSUPPORTED",
                3: "FIPA_ERR_WORKSPACE", 4: "FIPA_ERR_CUDA", 5: "FIPA_ERR_DEVICE_TIMEOUT",
                6: "FIPA_ERR_INTERNAL"}
F32, BF16 = 0, 1
DIM_FIELDS = ("B", "N", "H", "D", "Dv", "P", "Q", "Cz", "R", "Cout")


class FipaDims(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int) for f in DIM_FIELDS]


GRAD_FIELDS = ("q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "Wb", "point_w_raw",
               "w_out", "b_out")


class FipaGrads(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in GRAD_FIELDS]


class FipaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libfipa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libfipa.so not found at {_LIB_PATH}; build it with "
                           "`python -m protein_structure_models_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, c_int, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.fipa_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(FipaDims), c_int, c_int]
    lib.fipa_create.restype = c_int
    lib.fipa_workspace_size.argtypes = [vp, ctypes.POINTER(FipaDims), ctypes.POINTER(sz)]
    lib.fipa_workspace_size.restype = c_int
    lib.fipa_forward.argtypes = [vp] + [vp] * 12 + [vp, vp] + [vp, vp, ctypes.c_double,
                                                                ctypes.POINTER(FipaDims)] \
        + [vp] * 4 + [vp, sz, vp]
    lib.fipa_forward.restype = c_int
    lib.fipa_forward_rows.argtypes = [vp] + [vp] * 12 + [vp, vp] + [vp, vp, ctypes.c_double,
                                                                     ctypes.POINTER(FipaDims), c_int, c_int] \
        + [vp] * 4 + [vp, sz, vp]
    lib.fipa_forward_rows.restype = c_int
    lib.fipa_sync_status.argtypes = [vp, vp]
    lib.fipa_sync_status.restype = c_int
    lib.fipa_selftest_timeout.argtypes = [vp, ctypes.c_uint, vp]
    lib.fipa_selftest_timeout.restype = c_int
    lib.fipa_status_string.argtypes = [c_int]
    lib.fipa_status_string.restype = ctypes.c_char_p
    lib.fipa_last_error.argtypes = [vp]
    lib.fipa_last_error.restype = ctypes.c_char_p
    lib.fipa_enable_stage_timing.argtypes = [vp, c_int]
    lib.fipa_enable_stage_timing.restype = c_int
    lib.fipa_stage_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float), c_int]
    lib.fipa_stage_times.restype = c_int
    lib.fipa_trace_copy.argtypes = [vp, ctypes.POINTER(ctypes.c_int64), sz, vp]
    lib.fipa_trace_copy.restype = c_int
    lib.fipa_kernel_count.argtypes = [vp, ctypes.POINTER(FipaDims), c_int, ctypes.POINTER(c_int)]
    lib.fipa_kernel_count.restype = c_int
    lib.fipa_forward_noalloc.argtypes = [c_int] + [vp] * 12 + [vp, vp] + [vp, vp, ctypes.c_double,
                                                                         ctypes.POINTER(FipaDims)] \
        + [vp] * 3 + [vp]
    lib.fipa_forward_noalloc.restype = c_int
    lib.fipa_backward_workspace_size.argtypes = [vp, ctypes.POINTER(FipaDims), ctypes.POINTER(sz)]
    lib.fipa_backward_workspace_size.restype = c_int
    lib.fipa_backward.argtypes = [vp] + [vp] * 12 + [vp, vp] + [vp, vp, ctypes.c_double, ctypes.POINTER(FipaDims)] \
        + [vp, vp, ctypes.POINTER(FipaGrads), vp, sz, vp]
    lib.fipa_backward.restype = c_int
    lib.fipa_backward_saved.argtypes = lib.fipa_backward.argtypes
    lib.fipa_backward_saved.restype = c_int
    lib.fipa_forward_train.argtypes = [vp] + [vp] * 12 + [vp, vp] + [vp, vp, ctypes.c_double,
                                                                      ctypes.POINTER(FipaDims)] + [vp] * 3 + [vp, sz, vp]
    lib.fipa_forward_train.restype = c_int
    lib.fipa_backward_stage_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float), c_int]
    lib.fipa_backward_stage_times.restype = c_int
    lib.fipa_knn_distogram.argtypes = [c_int, vp, vp, c_int, c_int, c_int, vp, c_int, vp, vp, vp, vp, vp]
    lib.fipa_knn_distogram.restype = c_int
    lib.fipa_layer_workspace_size.argtypes = [vp, ctypes.POINTER(FipaDims), ctypes.POINTER(sz)]
    lib.fipa_layer_workspace_size.restype = c_int
    lib.fipa_ipa_layer.argtypes = [vp] + [vp] * 5 + [vp, vp] + [vp] * 6 + [ctypes.c_double, ctypes.POINTER(FipaDims)] \
        + [vp] * 4 + [vp, sz, vp]
    lib.fipa_ipa_layer.restype = c_int
    lib.fipa_destroy.argtypes = [vp]
    lib.fipa_destroy.restype = c_int
    _lib = lib
    return lib


def make_dims(**kw) -> FipaDims:
    return FipaDims(*[int(kw[f]) for f in DIM_FIELDS])


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


INPUT_KEYS = ("q", "k", "v", "q_points", "k_points", "v_points", "rotation", "translation",
              "z1", "z2", "Wb", "point_weight_raw")


class Fipa:
    """One library handle (one device, one input dtype)."""

    def __init__(self, dtype: str = "bf16", device: int = 0, max_dims: Optional[dict] = None):
        self.lib = load_library()
        self.dtype = dtype
        self.torch_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.device = device
        h = ctypes.c_void_p()
        md = make_dims(**max_dims) if max_dims else None
        st = self.lib.fipa_create(ctypes.byref(h), ctypes.byref(md) if md else None,
                                  BF16 if dtype == "bf16" else F32, device)
        if st != FIPA_OK:
            raise FipaError(st, "fipa_create failed")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            self.lib.fipa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st):
        if st != FIPA_OK:
            raise FipaError(st, self.lib.fipa_last_error(self.handle).decode())

    def workspace_size(self, dims: dict) -> int:
        d = make_dims(**dims)
        n = ctypes.c_size_t()
        self._check(self.lib.fipa_workspace_size(self.handle, ctypes.byref(d), ctypes.byref(n)))
        return int(n.value)

    TRACE_CAP = 4096

    def trace(self, stream: Optional[torch.cuda.Stream] = None):
        """Debug event log of the traced core CTA (needs FIPA_TRACE_CTA at creation):
        int64 array [4 roles, TRACE_CAP, 2] of (event id, SM clock), -1 = unused."""
        import numpy as np
        s = stream if stream is not None else torch.cuda.current_stream(torch.device("cuda", self.device))
        buf = np.empty((4, self.TRACE_CAP, 2), dtype=np.int64)
        self._check(self.lib.fipa_trace_copy(self.handle, buf.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                             buf.size, ctypes.c_void_p(s.cuda_stream)))
        return buf

    def kernel_count(self, dims: dict, with_attention: bool = False) -> int:
        d = make_dims(**dims)
        n = ctypes.c_int()
        self._check(self.lib.fipa_kernel_count(self.handle, ctypes.byref(d), 1 if with_attention else 0,
                                               ctypes.byref(n)))
        return int(n.value)

    def dims_of(self, inp: dict) -> dict:
        B, N, H, D = inp["q"].shape
        return dict(B=B, N=N, H=H, D=D, Dv=inp["v"].shape[-1], P=inp["q_points"].shape[3],
                    Q=inp["v_points"].shape[3], Cz=inp["z1"].shape[3], R=inp["z1"].shape[2],
                    Cout=inp["w_out"].shape[1])

    def forward(self, inp: dict, eps: float = 1e-8, want_attention: bool = False,
                want_lse: bool = False, workspace: Optional[torch.Tensor] = None,
                out: Optional[dict] = None, stream: Optional[torch.cuda.Stream] = None,
                rows: Optional[tuple] = None) -> dict:
        """Run fipa_forward on torch tensors (see workloads.make_inputs for keys/layouts).

        rows=(row_begin, row_end): fipa_forward_rows, only those query rows of every
        sample (the other rows of the outputs are left as they were)."""
        dev = torch.device("cuda", self.device)
        for k in INPUT_KEYS + ("w_out", "b_out"):
            t = inp[k]
            if t.dtype != self.torch_dtype or t.device != dev or not t.is_contiguous():
                raise ValueError(f"{k}: need a contiguous {self.torch_dtype} tensor on {dev}")
        mask = inp["mask"]
        pair_mask = inp.get("pair_mask")
        for name, t in (("mask", mask), ("pair_mask", pair_mask)):
            if t is not None and (t.dtype not in (torch.bool, torch.uint8) or t.device != dev
                                  or not t.is_contiguous()):
                raise ValueError(f"{name}: need a contiguous bool/uint8 tensor on {dev}")
        dims = self.dims_of(inp)
        B, N, H, Q, Cout = dims["B"], dims["N"], dims["H"], dims["Q"], dims["Cout"]
        if out is None:
            out = {"update": torch.empty((B, N, Cout), dtype=torch.float32, device=dev),
                   "local_points": torch.empty((B, N, H, Q, 3), dtype=torch.float32, device=dev)}
            if want_attention:
                out["attention"] = torch.empty((B, H, N, N), dtype=torch.float32, device=dev)
            if want_lse:
                out["lse"] = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        if workspace is None:
            workspace = torch.empty(self.workspace_size(dims), dtype=torch.uint8, device=dev)
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        d = make_dims(**dims)
        head = (self.handle, *[_ptr(inp[k]) for k in INPUT_KEYS], _ptr(mask), _ptr(pair_mask),
                _ptr(inp["w_out"]), _ptr(inp["b_out"]), float(eps), ctypes.byref(d))
        tail = (_ptr(out["update"]), _ptr(out["local_points"]), _ptr(out.get("attention")),
                _ptr(out.get("lse")), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                ctypes.c_void_p(s.cuda_stream))
        if rows is None:
            st = self.lib.fipa_forward(*head, *tail)
        else:
            st = self.lib.fipa_forward_rows(*head, int(rows[0]), int(rows[1]), *tail)
        self._check(st)
        return out

    # input key of each gradient (fipa_grads field -> workloads key)
    GRAD_KEYS = {"q": "q", "k": "k", "v": "v", "q_pts": "q_points", "k_pts": "k_points", "v_pts": "v_points",
                 "rot": "rotation", "trans": "translation", "z1": "z1", "z2": "z2", "Wb": "Wb",
                 "point_w_raw": "point_weight_raw", "w_out": "w_out", "b_out": "b_out"}

    def backward_workspace_size(self, dims: dict) -> int:
        d = make_dims(**dims)
        n = ctypes.c_size_t()
        self._check(self.lib.fipa_backward_workspace_size(self.handle, ctypes.byref(d), ctypes.byref(n)))
        return int(n.value)

    def forward_train(self, inp: dict, workspace: torch.Tensor, eps: float = 1e-8, out: Optional[dict] = None,
                      want_lse: bool = False, stream: Optional[torch.cuda.Stream] = None) -> dict:
        """fipa_forward_train: the forward, keeping in `workspace` (backward-sized)
        the state backward(..., saved=True) uses instead of a recompute."""
        dev = torch.device("cuda", self.device)
        dims = self.dims_of(inp)
        B, N, H, Q, Cout = dims["B"], dims["N"], dims["H"], dims["Q"], dims["Cout"]
        if out is None:
            out = {"update": torch.empty((B, N, Cout), dtype=torch.float32, device=dev),
                   "local_points": torch.empty((B, N, H, Q, 3), dtype=torch.float32, device=dev)}
            if want_lse:
                out["lse"] = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        d = make_dims(**dims)
        self._check(self.lib.fipa_forward_train(
            self.handle, *[_ptr(inp[k]) for k in INPUT_KEYS], _ptr(inp["mask"]), _ptr(inp.get("pair_mask")),
            _ptr(inp["w_out"]), _ptr(inp["b_out"]), float(eps), ctypes.byref(d), _ptr(out["update"]),
            _ptr(out["local_points"]), _ptr(out.get("lse")), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
            ctypes.c_void_p(s.cuda_stream)))
        return out

    def backward(self, inp: dict, d_update: torch.Tensor, d_local: Optional[torch.Tensor] = None,
                 eps: float = 1e-8, workspace: Optional[torch.Tensor] = None, grads: Optional[dict] = None,
                 stream: Optional[torch.cuda.Stream] = None, saved: bool = False) -> dict:
        """fipa_backward: float32 gradients of <d_update, update> + <d_local, local_points>
        for every floating input, keyed like the inputs (see workloads.make_inputs).
        saved=True: fipa_backward_saved, from the state a forward_train call left in
        `workspace` (no recompute)."""
        dev = torch.device("cuda", self.device)
        for k in INPUT_KEYS + ("w_out", "b_out"):
            t = inp[k]
            if t.dtype != self.torch_dtype or t.device != dev or not t.is_contiguous():
                raise ValueError(f"{k}: need a contiguous {self.torch_dtype} tensor on {dev}")
        for name, t in (("d_update", d_update), ("d_local", d_local)):
            if t is not None and (t.dtype != torch.float32 or t.device != dev or not t.is_contiguous()):
                raise ValueError(f"{name}: need a contiguous float32 tensor on {dev}")
        dims = self.dims_of(inp)
        if grads is None:
            grads = {key: torch.empty(inp[key].shape, dtype=torch.float32, device=dev)
                     for key in self.GRAD_KEYS.values()}
        if workspace is None:
            workspace = torch.empty(self.backward_workspace_size(dims), dtype=torch.uint8, device=dev)
        gs = FipaGrads(*[grads[self.GRAD_KEYS[f]].data_ptr() for f in GRAD_FIELDS])
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        d = make_dims(**dims)
        if saved and workspace is None:
            raise ValueError("saved=True needs the workspace of a forward_train call")
        fn = self.lib.fipa_backward_saved if saved else self.lib.fipa_backward
        st = fn(self.handle, *[_ptr(inp[k]) for k in INPUT_KEYS], _ptr(inp["mask"]),
                                    _ptr(inp.get("pair_mask")), _ptr(inp["w_out"]), _ptr(inp["b_out"]),
                                    float(eps), ctypes.byref(d), _ptr(d_update), _ptr(d_local), ctypes.byref(gs),
                                    _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                    ctypes.c_void_p(s.cuda_stream))
        self._check(st)
        return grads

    def ipa_layer(self, inp: dict, dims: dict, eps: float = 1e-8, workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> dict:
        """fipa_ipa_layer (float32 handle): the projection, the core, the residual and
        the frame update.  inp: s, W_in, b_in, rotation, translation, mask, pair_mask,
        Wb, point_weight_raw, w_out, b_out, W_bb, b_bb (float32 CUDA tensors, masks
        bool/uint8); dims: H, D, Dv, P, Q, Cz, R.  Returns s, rotation, translation,
        local_points."""
        dev = torch.device("cuda", self.device)
        s = inp["s"]
        B, N, Cs = s.shape
        full = dict(B=B, N=N, Cout=Cs, **{k: dims[k] for k in ("H", "D", "Dv", "P", "Q", "Cz", "R")})
        for k in ("s", "W_in", "b_in", "rotation", "translation", "Wb", "point_weight_raw", "w_out", "b_out",
                  "W_bb", "b_bb"):
            t = inp[k]
            if t.dtype != torch.float32 or t.device != dev or not t.is_contiguous():
                raise ValueError(f"{k}: need a contiguous float32 tensor on {dev}")
        d = make_dims(**full)
        if workspace is None:
            n = ctypes.c_size_t()
            self._check(self.lib.fipa_layer_workspace_size(self.handle, ctypes.byref(d), ctypes.byref(n)))
            workspace = torch.empty(int(n.value), dtype=torch.uint8, device=dev)
        out = {"s": torch.empty_like(s), "rotation": torch.empty_like(inp["rotation"]),
               "translation": torch.empty_like(inp["translation"]),
               "local_points": torch.empty((B, N, dims["H"], dims["Q"], 3), dtype=torch.float32, device=dev)}
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        self._check(self.lib.fipa_ipa_layer(
            self.handle, _ptr(s), _ptr(inp["W_in"]), _ptr(inp["b_in"]), _ptr(inp["rotation"]),
            _ptr(inp["translation"]), _ptr(inp["mask"]), _ptr(inp.get("pair_mask")), _ptr(inp["Wb"]),
            _ptr(inp["point_weight_raw"]), _ptr(inp["w_out"]), _ptr(inp["b_out"]), _ptr(inp["W_bb"]),
            _ptr(inp["b_bb"]), float(eps), ctypes.byref(d), _ptr(out["s"]), _ptr(out["rotation"]),
            _ptr(out["translation"]), _ptr(out["local_points"]), _ptr(workspace),
            ctypes.c_size_t(workspace.numel()), ctypes.c_void_p(st.cuda_stream)))
        return out

    BWD_STAGES = ("recompute", "prep", "q_side", "k_side", "chain")

    def backward_stage_times(self) -> dict:
        """Device ms of each stage of the most recent timed backward."""
        buf = (ctypes.c_float * len(self.BWD_STAGES))()
        self._check(self.lib.fipa_backward_stage_times(self.handle, buf, len(self.BWD_STAGES)))
        return dict(zip(self.BWD_STAGES, [float(x) for x in buf]))

    STAGES = ("prologue", "core", "out_proj", "attention")

    def enable_stage_timing(self, enable: bool = True):
        self._check(self.lib.fipa_enable_stage_timing(self.handle, 1 if enable else 0))

    def stage_times(self) -> dict:
        """Device ms of each stage of the most recent timed forward."""
        buf = (ctypes.c_float * len(self.STAGES))()
        self._check(self.lib.fipa_stage_times(self.handle, buf, len(self.STAGES)))
        return dict(zip(self.STAGES, [float(x) for x in buf]))

    def sync_status(self, stream: Optional[torch.cuda.Stream] = None):
        s = stream if stream is not None else torch.cuda.current_stream(torch.device("cuda", self.device))
        self._check(self.lib.fipa_sync_status(self.handle, ctypes.c_void_p(s.cuda_stream)))

    def selftest_timeout(self, timeout_ms: int, stream: Optional[torch.cuda.Stream] = None):
        """Launch the failure-path self-test (a bounded wait that runs out)."""
        s = stream if stream is not None else torch.cuda.current_stream(torch.device("cuda", self.device))
        self._check(self.lib.fipa_selftest_timeout(self.handle, int(timeout_ms), ctypes.c_void_p(s.cuda_stream)))


NOALLOC_SCRATCH_BYTES = 32 << 20


def forward_noalloc(inp: dict, eps: float = 1e-8, out: Optional[dict] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> dict:
    """fipa_forward_noalloc: the forward without a handle or a workspace, for
    callers that may not allocate device memory where they run it (a plugin
    whose host framework owns every device allocation, or a latency-bound
    caller that may not call cudaMalloc mid-step).  Its scratch is a fixed
    32 MiB device array inside the library; `out`, if given, must hold
    preallocated "update" and "local_points" (and optionally "lse") tensors,
    so this path allocates nothing either.  The call runs with the inputs'
    device made current, as the C entry point requires."""
    lib = load_library()
    q = inp["q"]
    dtype = BF16 if q.dtype == torch.bfloat16 else F32
    B, N, H, D = q.shape
    dims = dict(B=B, N=N, H=H, D=D, Dv=inp["v"].shape[-1], P=inp["q_points"].shape[3],
                Q=inp["v_points"].shape[3], Cz=inp["z1"].shape[3], R=inp["z1"].shape[2],
                Cout=inp["w_out"].shape[1])
    with torch.cuda.device(q.device):
        if out is None:
            out = {"update": torch.empty((B, N, dims["Cout"]), dtype=torch.float32, device=q.device),
                   "local_points": torch.empty((B, N, H, dims["Q"], 3), dtype=torch.float32, device=q.device)}
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        d = make_dims(**dims)
        st = lib.fipa_forward_noalloc(
            dtype, *[_ptr(inp[k]) for k in INPUT_KEYS], _ptr(inp["mask"]), _ptr(inp.get("pair_mask")),
            _ptr(inp["w_out"]), _ptr(inp["b_out"]), float(eps), ctypes.byref(d),
            _ptr(out["update"]), _ptr(out["local_points"]), _ptr(out.get("lse")),
            ctypes.c_void_p(s.cuda_stream))
    if st != FIPA_OK:
        raise FipaError(st, "fipa_forward_noalloc failed")
    return out


def knn_distogram(translation: torch.Tensor, mask: torch.Tensor, k: int, edges: torch.Tensor,
                  onehot: bool = True, out: Optional[dict] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> dict:
    """fipa_knn_distogram: the k nearest valid residues of every residue (self
    included, ties to the smaller index) and their distogram bins.
    translation [B,N,3] float32/bfloat16, mask [B,N] bool/uint8, edges
    [n_bins - 1] float32 ascending, all on one CUDA device.  Returns idx [B,N,k]
    int32, dist [B,N,k] float32, bin [B,N,k] int32 and (with onehot)
    onehot [B,N,k,n_bins] float32."""
    lib = load_library()
    dev = translation.device
    B, N, _ = translation.shape
    n_bins = edges.numel() + 1
    for name, t in (("translation", translation), ("mask", mask), ("edges", edges)):
        if t.device != dev or not t.is_contiguous():
            raise ValueError(f"{name}: need a contiguous tensor on {dev}")
    if translation.dtype not in (torch.float32, torch.bfloat16) or edges.dtype != torch.float32:
        raise ValueError("translation must be float32 or bfloat16, edges float32")
    with torch.cuda.device(dev):
        if out is None:
            out = {"idx": torch.empty((B, N, k), dtype=torch.int32, device=dev),
                   "dist": torch.empty((B, N, k), dtype=torch.float32, device=dev),
                   "bin": torch.empty((B, N, k), dtype=torch.int32, device=dev)}
            if onehot:
                out["onehot"] = torch.empty((B, N, k, n_bins), dtype=torch.float32, device=dev)
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        st = lib.fipa_knn_distogram(F32 if translation.dtype == torch.float32 else BF16, _ptr(translation),
                                    _ptr(mask), B, N, k, _ptr(edges) if edges.numel() else None, n_bins,
                                    _ptr(out["idx"]), _ptr(out["dist"]), _ptr(out["bin"]), _ptr(out.get("onehot")),
                                    ctypes.c_void_p(s.cuda_stream))
    if st != FIPA_OK:
        raise FipaError(st, "fipa_knn_distogram failed")
    return out


_handles: dict = {}


def invariant_point_attention(activations: dict, parameters: dict, masks: dict, structure: dict,
                              eps: float = 1e-8, return_attention: bool = True) -> dict:
    """The page's function signature, with the pair representation given as factors.

    activations: q, k, v, q_points, k_points, v_points, z1, z2
    parameters:  point_weight_raw, Wb, w_out, b_out
    masks:       mask, pair_mask (optional)
    structure:   rotation, translation
    Returns {"update", "local_points"} (+ "attention" when return_attention)."""
    inp = dict(activations)
    inp.update(parameters)
    inp.update(structure)
    inp["mask"] = masks["mask"]
    inp["pair_mask"] = masks.get("pair_mask")
    dt = "bf16" if inp["q"].dtype == torch.bfloat16 else "f32"
    dev = inp["q"].device.index or 0
    key = (dt, dev)
    if key not in _handles:
        _handles[key] = Fipa(dt, dev)
    h = _handles[key]
    out = h.forward(inp, eps=eps, want_attention=return_attention)
    return out
