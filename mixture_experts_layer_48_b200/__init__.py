"""Python binding of the B200 MoE layer library (libmoe.so, C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  The module refuses to load without
the compiled library -- there is no CPU fallback.

    from mixture_experts_layer_48_b200 import Moe
    layer = Moe(E=32, H=2880, I=2880, k=4)
    out = layer.forward(x, W_router, b_router, W_gate_up, W_down)   # out [T, H] fp32
    r = layer.route(x, W_router, b_router)   # topk_idx, topk_w, expert_offsets, perm, inv_perm
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python mixture_experts_layer_48_b200/build.py` "
        "(or __graft_entry__.build()); this package has no fallback")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE = 4, 5, 6
MOE_PATH_AUTO, MOE_PATH_STREAM, MOE_PATH_GEMM, MOE_PATH_TILE = 0, 1, 2, 3
MOE_PROFILE_KINDS = 10

# Every entry point of include/moe.h: name -> (restype, argtypes)
_c_int, _vp, _sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
_SIGS = {
    "moe_create": (_c_int, [_c_int, _c_int, _c_int, _c_int, ctypes.POINTER(_vp)]),
    "moe_destroy": (_c_int, [_vp]),
    "moe_workspace_bytes": (_sz, [_vp, _c_int]),
    "moe_route_workspace_bytes": (_sz, [_vp, _c_int]),
    "moe_route": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_forward": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_workspace_bytes_mxfp4": (_sz, [_vp, _c_int]),
    "moe_forward_mxfp4": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _sz, _vp]),
    "moe_set_path": (_c_int, [_vp, _c_int, _c_int]),
    "moe_get_path": (_c_int, [_vp, ctypes.POINTER(_c_int), ctypes.POINTER(_c_int)]),
    "moe_set_dispatch": (_c_int, [_vp, _c_int, _c_int, _c_int]),
    "moe_get_dispatch": (_c_int, [_vp, ctypes.POINTER(_c_int), ctypes.POINTER(_c_int),
                                  ctypes.POINTER(_c_int)]),
    "moe_tune_workspace_bytes": (_sz, [_vp, _c_int]),
    "moe_tune": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                          ctypes.POINTER(_c_int)]),
    "moe_sync_status": (_c_int, [_vp, _vp]),
    "moe_status_string": (ctypes.c_char_p, [_c_int]),
    "moe_launch_count": (ctypes.c_uint64, [_vp]),
    "moe_profile_begin": (_c_int, [_vp, _c_int]),
    "moe_profile_end": (_c_int, [_vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_c_int),
                                 _c_int]),
    "moe_profile_kind_name": (ctypes.c_char_p, [_c_int]),
    "moe_selftest_timeout": (_c_int, [_vp, _c_int, _vp]),
    "moe_permute": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_experts_workspace_bytes": (_sz, [_vp, _c_int, _c_int]),
    "moe_experts": (_c_int, [_vp, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_combine": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp]),
    "moe_last_dispatch": (_c_int, [_vp, _c_int, _c_int, _vp, _sz, _vp, _vp]),
    "moe_route_static_max_bytes": (_sz, []),
    "moe_route_static": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args
    globals()[_name] = _f

EXPORTED = tuple(_SIGS)


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {moe_status_string(status).decode()} (status {status})")


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, what)


def _ptr(t: torch.Tensor | None, dtype: torch.dtype, name: str, shape=None) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


class Moe:
    """One MoE layer shape (E experts, hidden H, intermediate I, top-k) bound to the current device."""

    def __init__(self, E: int, H: int, I: int, k: int):
        self.E, self.H, self.I, self.k = E, H, I, k
        h = _vp()
        _check(moe_create(E, H, I, k, ctypes.byref(h)), "moe_create")
        self._h = h
        self._ws = None

    # -- lifetime --------------------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None):
            moe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    # -- settings --------------------------------------------------------------------
    def set_path(self, path: int, crossover_T: int = -1) -> None:
        """Path; crossover_T >= 0 also sets the largest call AUTO streams (see include/moe.h)."""
        _check(moe_set_path(self._h, path, crossover_T), "moe_set_path")

    def get_path(self) -> tuple[int, int]:
        p, c = _c_int(), _c_int()
        _check(moe_get_path(self._h, ctypes.byref(p), ctypes.byref(c)), "moe_get_path")
        return p.value, c.value

    def set_dispatch(self, stream_rows: int = -1, tile_rows: int = -1, per_expert: int = -1) -> None:
        """AUTO thresholds in rows of one expert and the per-expert switch (negative: keep);
        see include/moe.h."""
        _check(moe_set_dispatch(self._h, stream_rows, tile_rows, int(per_expert)),
               "moe_set_dispatch")

    def get_dispatch(self) -> tuple[int, int, bool]:
        """(stream_rows, tile_rows, per_expert)."""
        s_, t_, p_ = _c_int(), _c_int(), _c_int()
        _check(moe_get_dispatch(self._h, ctypes.byref(s_), ctypes.byref(t_), ctypes.byref(p_)),
               "moe_get_dispatch")
        return s_.value, t_.value, bool(p_.value)

    def workspace_bytes(self, T: int) -> int:
        return moe_workspace_bytes(self._h, T)

    def route_workspace_bytes(self, T: int) -> int:
        return moe_route_workspace_bytes(self._h, T)

    def _workspace(self, nbytes: int, device) -> torch.Tensor:
        if self._ws is None or self._ws.numel() < nbytes or self._ws.device != device:
            self._ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self._ws

    # -- the layer -------------------------------------------------------------------
    def route(self, x, W_router, b_router, stream=None, workspace=None) -> dict:
        T = x.shape[0]
        E, H, k = self.E, self.H, self.k
        dev = x.device
        out = dict(
            topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
            topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
            expert_offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
            perm=torch.empty((T * k,), dtype=torch.int32, device=dev),
            inv_perm=torch.empty((T, k), dtype=torch.int32, device=dev),
        )
        need = self.route_workspace_bytes(T)
        ws = self._workspace(need, dev) if workspace is None else workspace
        st = moe_route(self._h, T, _ptr(x, torch.bfloat16, "x", (T, H)),
                       _ptr(W_router, torch.bfloat16, "W_router", (H, E)),
                       _ptr(b_router, torch.float32, "b_router", (E,)),
                       out["topk_idx"].data_ptr(), out["topk_w"].data_ptr(),
                       out["expert_offsets"].data_ptr(), out["perm"].data_ptr(),
                       out["inv_perm"].data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
        _check(st, "moe_route")
        return out

    def forward(self, x, W_router, b_router, W_gate_up, W_down, out=None, stream=None,
                workspace=None) -> torch.Tensor:
        T = x.shape[0]
        E, H, I = self.E, self.H, self.I
        if out is None:
            out = torch.empty((T, H), dtype=torch.float32, device=x.device)
        need = self.workspace_bytes(T)
        ws = self._workspace(need, x.device) if workspace is None else workspace
        st = moe_forward(self._h, T, _ptr(x, torch.bfloat16, "x", (T, H)),
                         _ptr(W_router, torch.bfloat16, "W_router", (H, E)),
                         _ptr(b_router, torch.float32, "b_router", (E,)),
                         _ptr(W_gate_up, torch.bfloat16, "W_gate_up", (E, H, 2 * I)),
                         _ptr(W_down, torch.bfloat16, "W_down", (E, I, H)),
                         _ptr(out, torch.float32, "out", (T, H)),
                         ws.data_ptr(), ws.numel(), _stream(stream))
        _check(st, "moe_forward")
        return out

    __call__ = forward

    # -- expert parallelism: device work on either side of the exchange (include/moe.h) --
    def permute(self, x, r: dict, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
        """Rows in expert order and their routing weights, from moe_route's outputs."""
        T = x.shape[0]
        R = T * self.k
        x_perm = torch.empty((R, self.H), dtype=torch.bfloat16, device=x.device)
        row_w = torch.empty((R,), dtype=torch.float32, device=x.device)
        st = moe_permute(self._h, T, _ptr(x, torch.bfloat16, "x", (T, self.H)),
                         _ptr(r["perm"], torch.int32, "perm", (R,)),
                         _ptr(r["inv_perm"], torch.int32, "inv_perm", (T, self.k)),
                         _ptr(r["topk_w"], torch.float32, "topk_w", (T, self.k)),
                         x_perm.data_ptr(), row_w.data_ptr(), _stream(stream))
        _check(st, "moe_permute")
        return x_perm, row_w

    def experts(self, x_rows, row_w, seg_counts, W_gate_up, W_down, stream=None,
                workspace=None) -> torch.Tensor:
        """The expert half on rows grouped as seg_counts [S, E] segments (source-major)."""
        R = x_rows.shape[0]
        S = seg_counts.shape[0]
        y = torch.empty((R, self.H), dtype=torch.float32, device=x_rows.device)
        if R == 0:
            return y
        need = moe_experts_workspace_bytes(self._h, R, S)
        if need == 0:
            raise ValueError("moe_experts: unsupported R or S")
        ws = self._workspace(need, x_rows.device) if workspace is None else workspace
        st = moe_experts(self._h, R, S, _ptr(seg_counts, torch.int32, "seg_counts", (S, self.E)),
                         _ptr(x_rows, torch.bfloat16, "x_rows", (R, self.H)),
                         _ptr(row_w, torch.float32, "row_w", (R,)),
                         _ptr(W_gate_up, torch.bfloat16, "W_gate_up", (self.E, self.H, 2 * self.I)),
                         _ptr(W_down, torch.bfloat16, "W_down", (self.E, self.I, self.H)),
                         y.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
        _check(st, "moe_experts")
        return y

    def combine(self, inv_perm, y_rows, out=None, stream=None) -> torch.Tensor:
        """out[t] = sum_j y_rows[inv_perm[t, j]] (slot order)."""
        T = inv_perm.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.float32, device=y_rows.device)
        st = moe_combine(self._h, T, _ptr(inv_perm, torch.int32, "inv_perm", (T, self.k)),
                         _ptr(y_rows, torch.float32, "y_rows", (T * self.k, self.H)),
                         _ptr(out, torch.float32, "out", (T, self.H)), _stream(stream))
        _check(st, "moe_combine")
        return out

    def workspace_bytes_mxfp4(self, T: int) -> int:
        return moe_workspace_bytes_mxfp4(self._h, T)

    def forward_mxfp4(self, x, W_router, b_router, gu_codes, gu_scales, dn_codes, dn_scales,
                      out=None, stream=None, workspace=None) -> torch.Tensor:
        """The layer with MXFP4 experts (uint8 codes and E8M0 scales, see include/moe.h)."""
        T = x.shape[0]
        E, H, I = self.E, self.H, self.I
        if out is None:
            out = torch.empty((T, H), dtype=torch.float32, device=x.device)
        need = self.workspace_bytes_mxfp4(T)
        ws = self._workspace(need, x.device) if workspace is None else workspace
        st = moe_forward_mxfp4(self._h, T, _ptr(x, torch.bfloat16, "x", (T, H)),
                               _ptr(W_router, torch.bfloat16, "W_router", (H, E)),
                               _ptr(b_router, torch.float32, "b_router", (E,)),
                               _ptr(gu_codes, torch.uint8, "gu_codes", (E, 2 * I, H // 2)),
                               _ptr(gu_scales, torch.uint8, "gu_scales", (E, H // 32, 2 * I)),
                               _ptr(dn_codes, torch.uint8, "dn_codes", (E, H, I // 2)),
                               _ptr(dn_scales, torch.uint8, "dn_scales", (E, I // 32, H)),
                               _ptr(out, torch.float32, "out", (T, H)),
                               ws.data_ptr(), ws.numel(), _stream(stream))
        _check(st, "moe_forward_mxfp4")
        return out

    def tune(self, x, W_router, b_router, W_gate_up, W_down, stream=None) -> int:
        T = x.shape[0]
        out = torch.empty((T, self.H), dtype=torch.float32, device=x.device)
        need = moe_tune_workspace_bytes(self._h, T)
        ws = self._workspace(need, x.device)
        c = _c_int()
        st = moe_tune(self._h, T, _ptr(x, torch.bfloat16, "x"), _ptr(W_router, torch.bfloat16, "W_router"),
                      _ptr(b_router, torch.float32, "b_router"), _ptr(W_gate_up, torch.bfloat16, "W_gate_up"),
                      _ptr(W_down, torch.bfloat16, "W_down"), out.data_ptr(), ws.data_ptr(), ws.numel(),
                      _stream(stream), ctypes.byref(c))
        _check(st, "moe_tune")
        return c.value

    def last_dispatch(self, T: int, workspace=None, mxfp4: bool = False, stream=None) -> tuple:
        """Work-list entries per family (streaming, expert tiles, row tiles; -1: not launched)
        of the last forward call of T tokens on `workspace` (default: the layer's own)."""
        ws = self._ws if workspace is None else workspace
        out = (ctypes.c_int32 * 3)()
        _check(moe_last_dispatch(self._h, T, int(mxfp4), ws.data_ptr(), ws.numel(), out,
                                 _stream(stream)), "moe_last_dispatch")
        return tuple(out)

    # -- status and measurement --------------------------------------------------------
    def sync_status(self, stream=None) -> int:
        return moe_sync_status(self._h, _stream(stream))

    def launch_count(self) -> int:
        return moe_launch_count(self._h)

    def profile_begin(self, max_calls: int) -> None:
        _check(moe_profile_begin(self._h, max_calls), "moe_profile_begin")

    def profile_end(self) -> dict:
        ms = (ctypes.c_float * MOE_PROFILE_KINDS)()
        n = (_c_int * MOE_PROFILE_KINDS)()
        _check(moe_profile_end(self._h, ms, n, MOE_PROFILE_KINDS), "moe_profile_end")
        return {moe_profile_kind_name(i).decode(): (ms[i], n[i]) for i in range(MOE_PROFILE_KINDS)}

    def selftest_timeout(self, limit_us: int, stream=None) -> None:
        _check(moe_selftest_timeout(self._h, limit_us, _stream(stream)), "moe_selftest_timeout")
