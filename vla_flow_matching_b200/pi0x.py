"""Python binding of libpi0x (include/pi0x.h) — argument marshalling only.

Every step of the denoising loop runs in the library's CUDA kernels; this module
only converts numpy arrays / torch tensors to pointers and checks status codes.
It raises if the shared library is missing: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpi0x.so")

PI0X_OK, PI0X_EINVAL, PI0X_EUNSUPPORTED, PI0X_ENOMEM, PI0X_ECUDA, PI0X_ETIMEOUT, PI0X_EDEVICE = range(7)
PI0X_BF16, PI0X_FP32 = 0, 1
PI0X_DTYPE_BF16, PI0X_DTYPE_F32 = 0, 1

#: Every symbol include/pi0x.h declares.
EXPORTED = ["pi0x_create", "pi0x_sample", "pi0x_sync_status", "pi0x_launch_count",
            "pi0x_status_string", "pi0x_last_error", "pi0x_destroy", "pi0x_version",
            "pi0x_debug_gemm_bf16", "pi0x_debug_attention", "pi0x_profile_enable", "pi0x_profile_read",
            "pi0x_set_variant", "pi0x_attention_noalloc", "pi0x_uses_loop", "pi0x_debug_loop_stall",
            "pi0x_debug_set_loop"]

#: time grids of pi0x_set_variant
PI0X_TIME_PI0 = 0
PI0X_TIME_LINSPACE = 1

#: kernel classes of pi0x_profile_read
K_CLASSES = ["prep", "embed", "gemm", "norm", "rope", "attn", "geglu", "final", "loop"]


class Pi0xError(RuntimeError):
    def __init__(self, status: int, what: str):
        lib = load()
        msg = lib.pi0x_status_string(status).decode()
        detail = lib.pi0x_last_error().decode()
        super().__init__(f"{what}: {msg} ({status}){': ' + detail if detail else ''}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("width", "depth", "mlp_dim", "num_heads", "num_kv_heads", "head_dim",
                 "horizon", "action_dim", "state_dim", "precision")]


_LAYER_FIELDS = ("in_norm_w", "q_w", "k_w", "v_w", "o_w", "post_norm_w", "gate_w", "up_w", "down_w")


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _LAYER_FIELDS]


_TOP_FIELDS = ("state_proj_w", "state_proj_b", "action_in_w", "action_in_b", "time_in_w",
               "time_in_b", "time_out_w", "time_out_b", "action_out_w", "action_out_b",
               "final_norm_w")


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _TOP_FIELDS] + [
        ("layers", ctypes.POINTER(LayerWeights)), ("dtype", ctypes.c_int)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libpi0x.so (built in-tree by vla_flow_matching_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: run `python -m vla_flow_matching_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    lib.pi0x_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Weights),
                                ctypes.POINTER(ctypes.c_void_p)]
    lib.pi0x_create.restype = ctypes.c_int
    lib.pi0x_sample.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p),
                                ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p, ctypes.c_int,
                                ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                ctypes.c_void_p, ctypes.c_void_p]
    lib.pi0x_sample.restype = ctypes.c_int
    lib.pi0x_set_variant.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.pi0x_set_variant.restype = ctypes.c_int
    lib.pi0x_sync_status.argtypes = [ctypes.c_void_p]
    lib.pi0x_sync_status.restype = ctypes.c_int
    lib.pi0x_launch_count.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.pi0x_launch_count.restype = ctypes.c_long
    lib.pi0x_status_string.argtypes = [ctypes.c_int]
    lib.pi0x_status_string.restype = ctypes.c_char_p
    lib.pi0x_last_error.argtypes = []
    lib.pi0x_last_error.restype = ctypes.c_char_p
    lib.pi0x_destroy.argtypes = [ctypes.c_void_p]
    lib.pi0x_destroy.restype = None
    lib.pi0x_version.argtypes = []
    lib.pi0x_version.restype = ctypes.c_int
    lib.pi0x_debug_gemm_bf16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p]
    lib.pi0x_debug_gemm_bf16.restype = ctypes.c_int
    lib.pi0x_debug_attention.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5 + [ctypes.c_void_p] * 2
    lib.pi0x_debug_attention.restype = ctypes.c_int
    lib.pi0x_attention_noalloc.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2
    lib.pi0x_attention_noalloc.restype = ctypes.c_int
    lib.pi0x_uses_loop.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.pi0x_uses_loop.restype = ctypes.c_int
    lib.pi0x_debug_loop_stall.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_ulonglong]
    lib.pi0x_debug_loop_stall.restype = ctypes.c_int
    lib.pi0x_debug_set_loop.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.pi0x_debug_set_loop.restype = ctypes.c_int
    lib.pi0x_profile_enable.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.pi0x_profile_enable.restype = ctypes.c_int
    lib.pi0x_profile_read.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_long),
                                      ctypes.POINTER(ctypes.c_double)]
    lib.pi0x_profile_read.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a) -> int:
    """Data pointer of a numpy array (host) or a torch tensor (host or device)."""
    if a is None:
        return 0
    if hasattr(a, "data_ptr"):
        if not a.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return int(a.data_ptr())
    if isinstance(a, np.ndarray):
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError("array must be C-contiguous")
        return int(a.ctypes.data)
    raise TypeError(f"unsupported array type {type(a)}")


def _check(status: int, what: str):
    if status != PI0X_OK:
        raise Pi0xError(status, what)


def debug_gemm_bf16(A, Bw, D, bn: int = 128, splits: int = 1, stream: int = 0):
    """D = A @ Bw.T with the library's tcgen05 GEMM (device torch tensors: bf16, bf16, fp32)."""
    M, K = A.shape
    N = Bw.shape[0]
    _check(load().pi0x_debug_gemm_bf16(_ptr(A), _ptr(Bw), M, N, K, _ptr(D), bn, splits,
                                       ctypes.c_void_p(stream)), "pi0x_debug_gemm_bf16")
    return D


def debug_attention(q, ks, vs, prefix_k, prefix_v, mask, B, H, P, step0, out, impl=1, stream: int = 0):
    """One layer of suffix attention with the library's kernels (device torch tensors)."""
    _check(load().pi0x_debug_attention(_ptr(q), _ptr(ks), _ptr(vs), _ptr(prefix_k), _ptr(prefix_v), _ptr(mask),
                                       B, H, P, int(step0), int(impl), _ptr(out), ctypes.c_void_p(stream)),
           "pi0x_debug_attention")
    return out


def attention_noalloc(q, ks, vs, prefix_k, prefix_v, mask, B, H, P, step0, out, stream: int = 0):
    """The same attention through pi0x_attention_noalloc (no device allocation;
    scratch in the library's static device array)."""
    _check(load().pi0x_attention_noalloc(_ptr(q), _ptr(ks), _ptr(vs), _ptr(prefix_k), _ptr(prefix_v), _ptr(mask),
                                         B, H, P, int(step0), _ptr(out), ctypes.c_void_p(stream)),
           "pi0x_attention_noalloc")
    return out


class Sampler:
    """A pi0x handle: expert weights on the device plus the loop's workspace.

    ``weights`` follows :func:`vla_flow_matching_b200.synth.make_weights`: a dict of
    arrays (bf16 bits as uint16, or float32) with a ``"layers"`` list.
    """

    def __init__(self, dims, weights: dict, precision: int = PI0X_BF16):
        lib = load()
        self._lib = lib
        self.dims = dims
        self.precision = precision
        cfg = Config(dims.width, dims.depth, dims.mlp_dim, dims.num_heads, dims.num_kv_heads,
                     dims.head_dim, dims.horizon, dims.action_dim, dims.state_dim, precision)
        first = weights["state_proj_w"]
        dtype = PI0X_DTYPE_BF16 if np.asarray(first).dtype == np.uint16 else PI0X_DTYPE_F32
        keep = []

        def arr(a):
            a = np.ascontiguousarray(a, dtype=np.uint16 if dtype == PI0X_DTYPE_BF16 else np.float32)
            keep.append(a)
            return _ptr(a)

        layers = (LayerWeights * dims.depth)()
        for i, lw in enumerate(weights["layers"]):
            for n in _LAYER_FIELDS:
                setattr(layers[i], n, arr(lw[n]))
        w = Weights(*[arr(weights[n]) for n in _TOP_FIELDS],
                    ctypes.cast(layers, ctypes.POINTER(LayerWeights)), dtype)
        h = ctypes.c_void_p()
        _check(lib.pi0x_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)), "pi0x_create")
        self._h = h

    def launch_count(self, B: int, P: int, num_steps: int) -> int:
        return int(self._lib.pi0x_launch_count(self._h, B, P, num_steps))

    def uses_loop(self, B: int) -> bool:
        """True if calls with batch B run the persistent small-batch loop kernel."""
        return bool(self._lib.pi0x_uses_loop(self._h, int(B)))

    def debug_set_loop(self, enable: bool):
        """Allow (True, default) or forbid (False) the persistent loop (see pi0x_debug.h)."""
        _check(self._lib.pi0x_debug_set_loop(self._h, int(bool(enable))), "pi0x_debug_set_loop")

    def debug_loop_stall(self, stage: int, wait_ns: int):
        """Make the next loop call stall at `stage` (test hook, see pi0x_debug.h)."""
        _check(self._lib.pi0x_debug_loop_stall(self._h, int(stage), int(wait_ns)), "pi0x_debug_loop_stall")

    def sample(self, prefix_k: Sequence, prefix_v: Sequence, mask, state, x1, num_steps: int,
               x0=None, stream: Optional[int] = None):
        """Enqueue one call; arrays may be torch tensors (host or device) or numpy arrays.

        Returns ``x0`` (the given output, or a new tensor/array like ``x1``).
        """
        if x0 is None:
            x0 = x1.new_empty(x1.shape) if hasattr(x1, "new_empty") else np.empty_like(x1)
        B, P = int(mask.shape[0]), int(mask.shape[1])
        L = self.dims.depth
        if len(prefix_k) != L or len(prefix_v) != L:
            raise ValueError("one prefix K and V per layer is required")
        pk = (ctypes.c_void_p * L)(*[_ptr(k) for k in prefix_k])
        pv = (ctypes.c_void_p * L)(*[_ptr(v) for v in prefix_v])
        if stream is None:
            try:
                import torch
                stream = torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
            except ImportError:
                stream = 0
        _check(self._lib.pi0x_sample(self._h, pk, pv, _ptr(mask), B, P, _ptr(state), _ptr(x1),
                                     int(num_steps), _ptr(x0), ctypes.c_void_p(stream)),
               "pi0x_sample")
        return x0

    def set_variant(self, time_grid: int = PI0X_TIME_PI0, x_prediction: bool = False,
                    causal_actions: bool = False):
        """Solver / convention variant for later calls (see pi0x_set_variant)."""
        _check(self._lib.pi0x_set_variant(self._h, int(time_grid), int(bool(x_prediction)),
                                          int(bool(causal_actions))), "pi0x_set_variant")

    def profile(self, on: bool = True):
        _check(self._lib.pi0x_profile_enable(self._h, int(on)), "pi0x_profile_enable")

    def profile_read(self) -> dict:
        """{class: (launches, total_ms)} of the most recent profiled call."""
        out = {}
        for i, name in enumerate(K_CLASSES):
            n, ms = ctypes.c_long(), ctypes.c_double()
            _check(self._lib.pi0x_profile_read(self._h, i, ctypes.byref(n), ctypes.byref(ms)),
                   "pi0x_profile_read")
            out[name] = (int(n.value), float(ms.value))
        return out

    def sync(self):
        _check(self._lib.pi0x_sync_status(self._h), "pi0x_sync_status")

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pi0x_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
