"""Python binding of the B200 MoE layer library (``libmoe.so``, C ABI in
``include/moe.h``).

Argument marshalling only: every stage runs in the library's CUDA kernels.
Tensors are torch CUDA tensors (device memory and streams come from torch);
each call passes ``data_ptr()`` values and the current torch stream.  There is
no fallback: if the compiled library is missing or cannot load, importing the
binding's entry points raises.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libmoe.so")
HEADER = os.path.join(ROOT, "include", "moe.h")

MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
ACT_NONE, ACT_RELU, ACT_SWIGLU = 0, 1, 2
QUANT_NONE, QUANT_PER_TENSOR, QUANT_PER_CHANNEL, QUANT_MX = 0, 1, 2, 6
QUANT_PER_GROUP, QUANT_PER_BLOCK = 4, 5

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
          3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_BAD_INDEX",
          6: "MOE_ERR_DEVICE_TIMEOUT"}
DTYPE_CODE = {"f32": MOE_F32, "bf16": MOE_BF16, "e4m3": MOE_E4M3}
ACT_CODE = {"none": ACT_NONE, "relu": ACT_RELU, "swiglu": ACT_SWIGLU}


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


class LayerDesc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("F", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("act", ctypes.c_int), ("quant", ctypes.c_int)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_r", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("w1", ctypes.c_void_p), ("w3", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("w_scale", ctypes.c_float), ("w_channel_scales", ctypes.c_void_p),
                ("w_mx_scales", ctypes.c_void_p), ("w_group_scales", ctypes.c_void_p)]


_lib = None


def header_functions() -> list[str]:
    """Names of the functions ``include/moe.h`` declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(moe_[a-z0-9_]+)\s*\(",
                      text, flags=re.M)


def load(path: str = LIB_PATH):
    """Load (once) the compiled library and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmoe.so not built at {path}; run "
                          "`python -m top_routing_grouped_gemv_b200._build`")
    L = ctypes.CDLL(path)
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    sig = {
        "moe_plan_create": ([ctypes.POINTER(LayerDesc), ctypes.POINTER(LayerWeights),
                             ctypes.POINTER(P)], ctypes.c_int),
        "moe_plan_destroy": ([P], ctypes.c_int),
        "moe_plan_refresh_router": ([P, P], ctypes.c_int),
        "moe_workspace_size": ([P, ctypes.POINTER(sz)], ctypes.c_int),
        "moe_workspace_init": ([P, P, sz, P], ctypes.c_int),
        "moe_router_topk": ([P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_permute": ([P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_permute_noalloc": ([P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
        "moe_grouped_ffn": ([P, P, P, f32, P, P, P, sz, P], ctypes.c_int),
        "moe_unpermute_combine": ([P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_shared_matmul": ([P, P, i32, i32, P, i32, f32, P, f32, P, P, P], ctypes.c_int),
        "moe_forward": ([P, P, P, P, sz, P], ctypes.c_int),
        "moe_forward_routed": ([P, P, P, P, f32, P, P, P, sz, P], ctypes.c_int),
        "moe_permute_quant": ([P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_forward_routed_shared": ([P, P, P, P, f32, P, P, P, i32, f32, P, P, P, sz, P],
                                      ctypes.c_int),
        "moe_forward_routed_dynamic": ([P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_forward_routed_mx": ([P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_permute_mx": ([P, P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_grouped_ffn_mx": ([P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_forward_routed_group_scales": ([P, P, f32, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_grouped_ffn_group_scales": ([P, P, f32, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_permute_n": ([P, i32, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_grouped_ffn_n": ([P, i32, P, P, f32, P, P, P, sz, P], ctypes.c_int),
        "moe_unpermute_combine_n": ([P, i32, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_forward_host": ([P, P, P, P, sz, P], ctypes.c_int),
        "moe_forward_host_async": ([P, P, P, P, sz, P], ctypes.c_int),
        "moe_host_join": ([P, P], ctypes.c_int),
        "moe_read_device_status": ([P, P, P], ctypes.c_int),
        "moe_profile_enable": ([P, ctypes.c_int], ctypes.c_int),
        "moe_profile_read": ([P, ctypes.POINTER(f32), ctypes.POINTER(ctypes.c_char_p),
                              ctypes.c_int, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
        "moe_last_launch_count": ([P], ctypes.c_int),
        "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "moe_selftest_wait_timeout": ([P, sz, i32, P, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != 0:
        raise MoEError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class Plan:
    """An executor for one layer shape and one set of device weights.

    ``weights``: dict with torch CUDA tensors ``w_r`` (d, E) fp32, optional
    ``bias`` (E,), ``w1`` (E, F, d), ``w3`` (E, F, d) for SwiGLU, ``w2``
    (E, d, F), and float ``w_scale`` (e4m3); for e4m3, optional
    ``w_channel_scales`` (E, F) fp32 (per-channel), ``w_group_scales`` (E, F,
    d/128) fp32 (per-group), ``w_block_scales`` (E, ceil(F/128), d/128) fp32
    (per-block) or ``w_mx_scales`` (E, F, d/32) uint8 E8M0 (MX).  The tensors are kept alive by the plan (the
    library only records their addresses).
    """

    def __init__(self, N, d, E, K, F, dtype: str, act: str, weights: dict):
        self.lib = load()
        self.N, self.d, self.E, self.K, self.F = N, d, E, K, F
        self.dtype, self.act = dtype, act
        self.d_out = F if act == "none" else d
        self._keep = dict(weights)
        quant = QUANT_NONE
        if dtype == "e4m3":
            quant = QUANT_PER_TENSOR
            given = [(key, code) for key, code in (("w_channel_scales", QUANT_PER_CHANNEL),
                                                   ("w_mx_scales", QUANT_MX),
                                                   ("w_group_scales", QUANT_PER_GROUP),
                                                   ("w_block_scales", QUANT_PER_BLOCK))
                     if weights.get(key) is not None]
            if len(given) > 1:
                raise ValueError("one weight scale mode per plan, got "
                                 + ", ".join(k for k, _ in given))
            if given:
                quant = given[0][1]
        desc = LayerDesc(N, d, E, K, F, DTYPE_CODE[dtype], ACT_CODE[act], quant)
        w = LayerWeights(_ptr(weights.get("w_r")), _ptr(weights.get("bias")),
                         _ptr(weights.get("w1")), _ptr(weights.get("w3")),
                         _ptr(weights.get("w2")), float(weights.get("w_scale", 1.0)),
                         _ptr(weights.get("w_channel_scales")), _ptr(weights.get("w_mx_scales")),
                         _ptr(weights.get("w_group_scales", weights.get("w_block_scales"))))
        h = ctypes.c_void_p()
        _check(self.lib.moe_plan_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(h)),
               "moe_plan_create")
        self.handle = h
        n = ctypes.c_size_t()
        _check(self.lib.moe_workspace_size(self.handle, ctypes.byref(n)), "moe_workspace_size")
        self.workspace_bytes = n.value

    def close(self):
        if getattr(self, "handle", None):
            self.lib.moe_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def refresh_router(self, stream=None):
        """Re-derive the plan's copy of the router weights after w_r changed
        in place (moe_plan_refresh_router)."""
        _check(self.lib.moe_plan_refresh_router(self.handle, _stream(stream)),
               "moe_plan_refresh_router")

    # -- workspace ---------------------------------------------------------
    def new_workspace(self, device=None):
        import torch
        ws = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device or "cuda")
        _check(self.lib.moe_workspace_init(self.handle, _ptr(ws), ws.numel(), _stream()),
               "moe_workspace_init")
        return ws

    # -- stages ------------------------------------------------------------
    def router_topk(self, x, ids, gates, ws, margin=None, stream=None):
        _check(self.lib.moe_router_topk(self.handle, _ptr(x), _ptr(ids), _ptr(gates),
                                        _ptr(margin), _ptr(ws), ws.numel(), _stream(stream)),
               "moe_router_topk")

    def permute(self, x, ids, counts, offsets, pos, src, x_perm, ws, stream=None, n=None):
        """n: the number of tokens (default the plan's N)."""
        if n is None:
            _check(self.lib.moe_permute(self.handle, _ptr(x), _ptr(ids), _ptr(counts),
                                        _ptr(offsets), _ptr(pos), _ptr(src), _ptr(x_perm),
                                        _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
        else:
            _check(self.lib.moe_permute_n(self.handle, int(n), _ptr(x), _ptr(ids), _ptr(counts),
                                          _ptr(offsets), _ptr(pos), _ptr(src), _ptr(x_perm),
                                          _ptr(ws), ws.numel(), _stream(stream)), "moe_permute_n")

    def permute_noalloc(self, x, ids, counts, offsets, pos, src, x_perm, device_status=None,
                        stream=None):
        """moe_permute without a workspace (scratch in the library's static
        device memory; see include/moe.h)."""
        _check(self.lib.moe_permute_noalloc(self.handle, _ptr(x), _ptr(ids), _ptr(counts),
                                            _ptr(offsets), _ptr(pos), _ptr(src), _ptr(x_perm),
                                            _ptr(device_status), _stream(stream)),
               "moe_permute_noalloc")

    def grouped_ffn(self, x_perm, offsets, y_perm, ws, x_scale: float = 1.0, x_row_scales=None,
                    stream=None, n=None):
        if n is None:
            _check(self.lib.moe_grouped_ffn(self.handle, _ptr(x_perm), _ptr(offsets), x_scale,
                                            _ptr(x_row_scales), _ptr(y_perm), _ptr(ws), ws.numel(),
                                            _stream(stream)), "moe_grouped_ffn")
        else:
            _check(self.lib.moe_grouped_ffn_n(self.handle, int(n), _ptr(x_perm), _ptr(offsets),
                                              x_scale, _ptr(x_row_scales), _ptr(y_perm), _ptr(ws),
                                              ws.numel(), _stream(stream)), "moe_grouped_ffn_n")

    def unpermute_combine(self, y_perm, pos, gates, y, ws, stream=None, n=None):
        if n is None:
            _check(self.lib.moe_unpermute_combine(self.handle, _ptr(y_perm), _ptr(pos),
                                                  _ptr(gates), _ptr(y), _ptr(ws), ws.numel(),
                                                  _stream(stream)), "moe_unpermute_combine")
        else:
            _check(self.lib.moe_unpermute_combine_n(self.handle, int(n), _ptr(y_perm), _ptr(pos),
                                                    _ptr(gates), _ptr(y), _ptr(ws), ws.numel(),
                                                    _stream(stream)), "moe_unpermute_combine_n")

    def shared_matmul(self, x, w, x_scale, w_scale, y, x_token_scales=None,
                      w_channel_scales=None, stream=None):
        M, H = x.shape
        N2 = w.shape[0]
        _check(self.lib.moe_shared_matmul(self.handle, _ptr(x), M, H, _ptr(w), N2, x_scale,
                                          _ptr(x_token_scales), w_scale, _ptr(w_channel_scales),
                                          _ptr(y), _stream(stream)), "moe_shared_matmul")

    def forward(self, x, y, ws, stream=None):
        _check(self.lib.moe_forward(self.handle, _ptr(x), _ptr(y), _ptr(ws), ws.numel(),
                                    _stream(stream)), "moe_forward")

    def forward_routed(self, x, ids, gates, y, ws, x_scale: float = 1.0, x_token_scales=None,
                       stream=None):
        _check(self.lib.moe_forward_routed(self.handle, _ptr(x), _ptr(ids), _ptr(gates), x_scale,
                                           _ptr(x_token_scales), _ptr(y), _ptr(ws), ws.numel(),
                                           _stream(stream)), "moe_forward_routed")

    def permute_quant(self, x_bf16, ids, counts, offsets, pos, src, x_perm, token_scales, ws,
                      stream=None):
        _check(self.lib.moe_permute_quant(self.handle, _ptr(x_bf16), _ptr(ids), _ptr(counts),
                                          _ptr(offsets), _ptr(pos), _ptr(src), _ptr(x_perm),
                                          _ptr(token_scales), _ptr(ws), ws.numel(),
                                          _stream(stream)), "moe_permute_quant")

    def forward_routed_mx(self, x, x_mx_scales, ids, gates, y, ws, stream=None):
        _check(self.lib.moe_forward_routed_mx(self.handle, _ptr(x), _ptr(x_mx_scales), _ptr(ids),
                                              _ptr(gates), _ptr(y), _ptr(ws), ws.numel(),
                                              _stream(stream)), "moe_forward_routed_mx")

    def permute_mx(self, x, x_mx_scales, ids, counts, offsets, pos, src, x_perm,
                   x_perm_mx_scales, ws, stream=None):
        _check(self.lib.moe_permute_mx(self.handle, _ptr(x), _ptr(x_mx_scales), _ptr(ids),
                                       _ptr(counts), _ptr(offsets), _ptr(pos), _ptr(src),
                                       _ptr(x_perm), _ptr(x_perm_mx_scales), _ptr(ws), ws.numel(),
                                       _stream(stream)), "moe_permute_mx")

    def grouped_ffn_mx(self, x_perm, x_perm_mx_scales, offsets, y_perm, ws, stream=None):
        _check(self.lib.moe_grouped_ffn_mx(self.handle, _ptr(x_perm), _ptr(x_perm_mx_scales),
                                           _ptr(offsets), _ptr(y_perm), _ptr(ws), ws.numel(),
                                           _stream(stream)), "moe_grouped_ffn_mx")

    def forward_routed_group_scales(self, x, ids, gates, y, ws, x_scale: float = 1.0,
                                    x_token_scales=None, x_group_scales=None, stream=None):
        _check(self.lib.moe_forward_routed_group_scales(
            self.handle, _ptr(x), x_scale, _ptr(x_token_scales), _ptr(x_group_scales), _ptr(ids),
            _ptr(gates), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
            "moe_forward_routed_group_scales")

    def grouped_ffn_group_scales(self, x_perm, offsets, y_perm, ws, x_scale: float = 1.0,
                                 x_row_scales=None, x_group_scales=None, stream=None):
        _check(self.lib.moe_grouped_ffn_group_scales(
            self.handle, _ptr(x_perm), x_scale, _ptr(x_row_scales), _ptr(x_group_scales),
            _ptr(offsets), _ptr(y_perm), _ptr(ws), ws.numel(), _stream(stream)),
            "moe_grouped_ffn_group_scales")

    def forward_routed_dynamic(self, x_bf16, ids, gates, y, ws, stream=None):
        _check(self.lib.moe_forward_routed_dynamic(self.handle, _ptr(x_bf16), _ptr(ids),
                                                   _ptr(gates), _ptr(y), _ptr(ws), ws.numel(),
                                                   _stream(stream)), "moe_forward_routed_dynamic")

    def forward_routed_shared(self, x, ids, gates, y, w_sh, w_sh_scale, y_sh, ws,
                              x_scale: float = 1.0, x_token_scales=None,
                              w_sh_channel_scales=None, stream=None):
        _check(self.lib.moe_forward_routed_shared(
            self.handle, _ptr(x), _ptr(ids), _ptr(gates), x_scale, _ptr(x_token_scales), _ptr(y),
            _ptr(w_sh), w_sh.shape[0], w_sh_scale, _ptr(w_sh_channel_scales), _ptr(y_sh), _ptr(ws),
            ws.numel(), _stream(stream)), "moe_forward_routed_shared")

    def forward_host(self, x_host, y_host, ws, stream=None):
        _check(self.lib.moe_forward_host(self.handle, _ptr(x_host), _ptr(y_host), _ptr(ws),
                                         ws.numel(), _stream(stream)), "moe_forward_host")

    def forward_host_async(self, x_host, y_host, ws, stream=None):
        _check(self.lib.moe_forward_host_async(self.handle, _ptr(x_host), _ptr(y_host), _ptr(ws),
                                               ws.numel(), _stream(stream)),
               "moe_forward_host_async")

    def host_join(self, stream=None):
        _check(self.lib.moe_host_join(self.handle, _stream(stream)), "moe_host_join")

    def read_device_status(self, ws, stream=None) -> int:
        return self.lib.moe_read_device_status(self.handle, _ptr(ws), _stream(stream))

    # -- profiling ---------------------------------------------------------
    def profile(self, enable: bool = True):
        _check(self.lib.moe_profile_enable(self.handle, int(enable)), "moe_profile_enable")

    def profile_read(self) -> list[tuple[str, float]]:
        ms = (ctypes.c_float * 16)()
        names = (ctypes.c_char_p * 16)()
        n = ctypes.c_int()
        _check(self.lib.moe_profile_read(self.handle, ms, names, 16, ctypes.byref(n)),
               "moe_profile_read")
        return [(names[i].decode(), ms[i]) for i in range(n.value)]

    def last_launch_count(self) -> int:
        return self.lib.moe_last_launch_count(self.handle)


def selftest_wait_timeout(ws, limit_us: int, leave_order=None, stream=None):
    """Run the bounded-wait failure-path self-test (see include/moe.h)."""
    lib = load()
    _check(lib.moe_selftest_wait_timeout(_ptr(ws), ws.numel(), int(limit_us), _ptr(leave_order),
                                         _stream(stream)), "moe_selftest_wait_timeout")


def build(force: bool = False, verbose: bool = False) -> str:
    from . import _build
    return _build.build(force=force, verbose=verbose)
