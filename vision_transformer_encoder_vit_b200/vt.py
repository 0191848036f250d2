"""Thin ctypes binding of libvt (include/vt.h): argument marshalling only.

Every function here has the name of the C entry point it calls and passes plain
pointers and sizes; all computation happens in the library's CUDA kernels.  PyTorch
tensors are accepted for device buffers (their data_ptr() is passed) so that tests
and the benchmark can use torch for device memory and streams.

If libvt.so has not been built, importing this module raises ImportError: there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvt.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libvt.so is not built ({_LIB_PATH}); run "
                      "`python -m vision_transformer_encoder_vit_b200.build`")
lib = ctypes.CDLL(_LIB_PATH)

STATUS = {0: "VT_OK", 1: "VT_ERR_INVALID_ARG", 2: "VT_ERR_SHAPE", 3: "VT_ERR_NOT_LOADED",
          4: "VT_ERR_WEIGHT", 5: "VT_ERR_WORKSPACE", 6: "VT_ERR_UNSUPPORTED", 7: "VT_ERR_CUDA",
          8: "VT_ERR_TIMEOUT"}
STATUS_CODE = {v: k for k, v in STATUS.items()}

PROFILE_CLASSES = ("gemm", "attention", "layernorm", "patch_unfold", "reorder", "attention_prep",
                   "attention_backward", "backward_misc")


class VtError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name}: {vt_last_error()}")


class vt_config(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int), ("hidden", ctypes.c_int), ("heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("mlp", ctypes.c_int), ("patch", ctypes.c_int),
                ("temporal_patch", ctypes.c_int), ("merge", ctypes.c_int),
                ("rope_sections", ctypes.c_int * 3), ("rope_theta", ctypes.c_float),
                ("ln_eps", ctypes.c_float), ("gelu_tanh", ctypes.c_int),
                ("proj_gelu_tanh", ctypes.c_int), ("proj_hidden", ctypes.c_int),
                ("proj_out", ctypes.c_int), ("use_rope", ctypes.c_int)]


class vt_weight(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("data", ctypes.c_void_p), ("ndim", ctypes.c_int),
                ("shape", ctypes.c_int64 * 5)]


_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t
_i32p = ctypes.POINTER(ctypes.c_int32)
_fp = ctypes.POINTER(ctypes.c_float)

_SIGS = {
    "vt_create": ([ctypes.POINTER(vt_config), ctypes.POINTER(_vp)]),
    "vt_destroy": ([_vp]),
    "vt_load_weights": ([_vp, ctypes.POINTER(vt_weight), _i]),
    "vt_workspace_bytes": ([_vp, _i, _i32p, ctypes.POINTER(_sz)]),
    "vt_forward": ([_vp, _vp, _i32p, _i, _vp, _vp, _vp, _sz, _vp]),
    "vt_forward_host": ([_vp, _vp, _i32p, _i, _vp, _vp, _sz, _vp]),
    "vt_forward_host_workspace_bytes": ([_vp, _i, _i32p, ctypes.POINTER(_sz)]),
    "vt_forward_host_async": ([_vp, _vp, _i32p, _i, _vp, _vp, _sz, _vp]),
    "vt_workspace_bytes_varlen": ([_vp, _i, _i32p, ctypes.POINTER(_sz)]),
    "vt_forward_varlen": ([_vp, _vp, _i32p, _i, _vp, _vp, _vp, _sz, _vp]),
    "vt_forward_video": ([_vp, _vp, _i, _i32p, _i, _vp, _vp, _vp, _sz, _vp]),
    "vt_preprocess": ([_vp, _vp, _i32p, _i, _i32p, _fp, _fp, _vp, _vp]),
    "vt_enable_backward": ([_vp]),
    "vt_backward_bytes": ([_vp, _i, _i32p, ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "vt_forward_saved": ([_vp, _vp, _i32p, _i, _vp, _vp, _sz, _vp, _sz, _vp]),
    "vt_backward": ([_vp, _vp, _i32p, _i, _vp, _vp, _vp, _sz, _vp]),
    "vt_attention_backward_workspace_bytes": ([_i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "vt_attention_backward": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "vt_layernorm_backward": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _f, _vp]),
    "vt_forward_u8": ([_vp, _vp, _i32p, _i, _i32p, _fp, _fp, _vp, _vp, _vp, _sz, _vp]),
    "vt_tower_layer": ([_vp, _i, _vp, _vp, _i32p, _i, _vp, _sz, _vp]),
    "vt_tower_layer_backward_bytes": ([_vp, _i, _i32p, ctypes.POINTER(_sz)]),
    "vt_tower_layer_backward": ([_vp, _i, _vp, _vp, _vp, _i32p, _i, _vp, _sz, _vp]),
    "vt_patch_embed": ([_vp, _vp, _i32p, _i, _vp, _vp, _sz, _vp]),
    "vt_merge_project": ([_vp, _vp, _i32p, _i, _vp, _vp, _sz, _vp]),
    "vt_attention_workspace_bytes": ([_i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "vt_attention": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _i32p, _f, _f, _vp, _sz, _vp]),
    "vt_attention_prepared": ([_vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _f, _vp]),
    "vt_attention_static": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _i32p, _f, _f, _vp]),
    "vt_attention_static_max_bytes": ([ctypes.POINTER(_sz)]),
    "vt_linear": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "vt_linear_ws": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "vt_linear_workspace_bytes": ([ctypes.POINTER(_sz)]),
    "vt_layernorm": ([_vp, _vp, _vp, _vp, _i, _i, _f, _vp]),
    "vt_patch_unfold": ([_vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "vt_index_maps": ([_i32p, _i32p, _i32p, _i32p]),
    "vt_check": ([_vp]),
    "vt_selftest_wait_timeout": ([_vp]),
    "vt_profile_begin": ([_vp]),
    "vt_profile_end": ([_vp]),
    "vt_profile_read": ([_i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                         ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
    "vt_profile_launches": ([ctypes.POINTER(ctypes.c_int64)]),
    "vt_profile_launch": ([ctypes.c_int64, ctypes.POINTER(_i), ctypes.POINTER(ctypes.c_double),
                           ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
}
for _name, _args in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int
lib.vt_last_error.argtypes = []
lib.vt_last_error.restype = ctypes.c_char_p

EXPORTED = tuple(_SIGS) + ("vt_last_error",)


# ------------------------------------------------------------------ helpers

def _ptr(x) -> int | None:
    """Device pointer of a torch tensor (or an int / None passed through)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream
        except Exception:
            return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _grid(g) -> ctypes.Array:
    return (ctypes.c_int32 * 3)(*[int(v) for v in g])


def _check(status: int, where: str) -> None:
    if status != 0:
        raise VtError(status, where)


def vt_last_error() -> str:
    return lib.vt_last_error().decode()


def make_config(cfg: dict) -> vt_config:
    c = vt_config()
    c.layers, c.hidden, c.heads, c.head_dim = cfg["layers"], cfg["hidden"], cfg["heads"], cfg["head_dim"]
    c.mlp, c.patch, c.temporal_patch, c.merge = cfg["mlp"], cfg["patch"], cfg["temporal_patch"], cfg["merge"]
    for i, s in enumerate(cfg["rope_sections"]):
        c.rope_sections[i] = s
    c.rope_theta, c.ln_eps = cfg["rope_theta"], cfg["ln_eps"]
    c.gelu_tanh, c.proj_gelu_tanh = int(cfg["gelu_tanh"]), int(cfg["proj_gelu_tanh"])
    c.proj_hidden, c.proj_out = cfg["proj_hidden"], cfg["proj_out"]
    c.use_rope = int(cfg.get("use_rope", True))
    return c


# --------------------------------------------------------------- C calls

def vt_create(cfg: dict | vt_config) -> int:
    c = cfg if isinstance(cfg, vt_config) else make_config(cfg)
    h = _vp()
    _check(lib.vt_create(ctypes.byref(c), ctypes.byref(h)), "vt_create")
    return h.value


def vt_destroy(h: int) -> None:
    _check(lib.vt_destroy(h), "vt_destroy")


def vt_load_weights(h: int, tensors: dict) -> None:
    """tensors: name -> device bf16 tensor (kept alive by the caller)."""
    arr = (vt_weight * len(tensors))()
    names = []
    for i, (name, t) in enumerate(tensors.items()):
        nb = name.encode()
        names.append(nb)
        arr[i].name = nb
        arr[i].data = _ptr(t)
        arr[i].ndim = t.dim()
        for j, s in enumerate(t.shape):
            arr[i].shape[j] = int(s)
    _check(lib.vt_load_weights(h, arr, len(tensors)), "vt_load_weights")


def vt_workspace_bytes(h: int, B: int, grid_thw) -> int:
    out = _sz()
    _check(lib.vt_workspace_bytes(h, B, _grid(grid_thw), ctypes.byref(out)), "vt_workspace_bytes")
    return out.value


def vt_forward(h, pixels, grid_thw, B, out, tower_out, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_forward(h, _ptr(pixels), _grid(grid_thw), B, _ptr(out), _ptr(tower_out), _ptr(ws),
                          ws_bytes, _stream(stream)), "vt_forward")


def vt_forward_video(h, clips, frames, grid_thw, B, out, tower_out, ws, ws_bytes, stream=None) -> None:
    """clips: device fp32 [B, frames, 3, H, W]; grid_thw = (ceil(frames / tp), H/p, W/p)."""
    _check(lib.vt_forward_video(h, _ptr(clips), frames, _grid(grid_thw), B, _ptr(out), _ptr(tower_out), _ptr(ws),
                                ws_bytes, _stream(stream)), "vt_forward_video")


def _stats(v) -> ctypes.Array | None:
    return None if v is None else (ctypes.c_float * 3)(*[float(x) for x in v])


def _sizes(src_hw) -> ctypes.Array:
    flat = [int(v) for hw in src_hw for v in hw]
    return (ctypes.c_int32 * len(flat))(*flat)


def vt_preprocess(h, images, src_hw, grid_thw, pixels, mean=None, std=None, stream=None) -> None:
    """images: device uint8, the images' [H0, W0, 3] arrays concatenated; src_hw: list of
    (H0, W0); pixels: device fp32 [B, 3, h*p, w*p].  mean/std None: CLIP statistics."""
    _check(lib.vt_preprocess(h, _ptr(images), _sizes(src_hw), len(src_hw), _grid(grid_thw), _stats(mean),
                             _stats(std), _ptr(pixels), _stream(stream)), "vt_preprocess")


def vt_forward_u8(h, images, src_hw, grid_thw, out, tower_out, ws, ws_bytes, mean=None, std=None,
                  stream=None) -> None:
    _check(lib.vt_forward_u8(h, _ptr(images), _sizes(src_hw), len(src_hw), _grid(grid_thw), _stats(mean),
                             _stats(std), _ptr(out), _ptr(tower_out), _ptr(ws), ws_bytes, _stream(stream)),
           "vt_forward_u8")


def vt_enable_backward(h) -> None:
    _check(lib.vt_enable_backward(h), "vt_enable_backward")


def vt_backward_bytes(h, B, grid_thw) -> tuple[int, int]:
    """(saved-activation bytes, workspace bytes) of vt_forward_saved / vt_backward."""
    a, b = _sz(), _sz()
    _check(lib.vt_backward_bytes(h, B, _grid(grid_thw), ctypes.byref(a), ctypes.byref(b)), "vt_backward_bytes")
    return a.value, b.value


def vt_forward_saved(h, pixels, grid_thw, B, tower_out, saved, saved_bytes, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_forward_saved(h, _ptr(pixels), _grid(grid_thw), B, _ptr(tower_out), _ptr(saved), saved_bytes,
                                _ptr(ws), ws_bytes, _stream(stream)), "vt_forward_saved")


def vt_backward(h, saved, grid_thw, B, d_tower, d_pixels, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_backward(h, _ptr(saved), _grid(grid_thw), B, _ptr(d_tower), _ptr(d_pixels), _ptr(ws), ws_bytes,
                           _stream(stream)), "vt_backward")


def vt_attention_backward_workspace_bytes(B, H, N, D) -> int:
    out = _sz()
    _check(lib.vt_attention_backward_workspace_bytes(B, H, N, D, ctypes.byref(out)),
           "vt_attention_backward_workspace_bytes")
    return out.value


def vt_attention_backward(q, k, v, dO, dqkv, B, H, N, D, scale, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dqkv), B, H, N, D, scale, _ptr(ws),
                                     ws_bytes, _stream(stream)), "vt_attention_backward")


def vt_layernorm_backward(x, gamma, dy, dres, dx, rows, cols, eps, stream=None) -> None:
    _check(lib.vt_layernorm_backward(_ptr(x), _ptr(gamma), _ptr(dy), _ptr(dres), _ptr(dx), rows, cols, eps,
                                     _stream(stream)), "vt_layernorm_backward")


def _grids(grids) -> ctypes.Array:
    flat = [int(v) for g in grids for v in g]
    return (ctypes.c_int32 * len(flat))(*flat)


def vt_workspace_bytes_varlen(h: int, grids) -> int:
    out = _sz()
    _check(lib.vt_workspace_bytes_varlen(h, len(grids), _grids(grids), ctypes.byref(out)),
           "vt_workspace_bytes_varlen")
    return out.value


def vt_forward_varlen(h, pixels, grids, out, tower_out, ws, ws_bytes, stream=None) -> None:
    """grids: list of (t, h, w) per image; pixels: the images' [3, H, W] fp32 arrays
    concatenated on the device."""
    _check(lib.vt_forward_varlen(h, _ptr(pixels), _grids(grids), len(grids), _ptr(out), _ptr(tower_out), _ptr(ws),
                                 ws_bytes, _stream(stream)), "vt_forward_varlen")


def vt_forward_host_workspace_bytes(h: int, B: int, grid_thw) -> int:
    out = _sz()
    _check(lib.vt_forward_host_workspace_bytes(h, B, _grid(grid_thw), ctypes.byref(out)),
           "vt_forward_host_workspace_bytes")
    return out.value


def vt_forward_host(h, pixels_host, grid_thw, B, out_host, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_forward_host(h, _ptr(pixels_host), _grid(grid_thw), B, _ptr(out_host), _ptr(ws), ws_bytes,
                               _stream(stream)), "vt_forward_host")


def vt_forward_host_async(h, pixels_host, grid_thw, B, out_host, ws, ws_bytes, stream=None) -> None:
    """Enqueues vt_forward_host on `stream` without synchronising it."""
    _check(lib.vt_forward_host_async(h, _ptr(pixels_host), _grid(grid_thw), B, _ptr(out_host), _ptr(ws), ws_bytes,
                                     _stream(stream)), "vt_forward_host_async")


def vt_tower_layer(h, layer, x_in, x_out, grid_thw, B, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_tower_layer(h, layer, _ptr(x_in), _ptr(x_out), _grid(grid_thw), B, _ptr(ws), ws_bytes,
                              _stream(stream)), "vt_tower_layer")


def vt_tower_layer_backward_bytes(h, B, grid_thw) -> int:
    out = _sz()
    _check(lib.vt_tower_layer_backward_bytes(h, B, _grid(grid_thw), ctypes.byref(out)),
           "vt_tower_layer_backward_bytes")
    return out.value


def vt_tower_layer_backward(h, layer, x_in, dy, dx, grid_thw, B, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_tower_layer_backward(h, layer, _ptr(x_in), _ptr(dy), _ptr(dx), _grid(grid_thw), B, _ptr(ws),
                                       ws_bytes, _stream(stream)), "vt_tower_layer_backward")


def vt_patch_embed(h, pixels, grid_thw, B, x_out, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_patch_embed(h, _ptr(pixels), _grid(grid_thw), B, _ptr(x_out), _ptr(ws), ws_bytes,
                              _stream(stream)), "vt_patch_embed")


def vt_merge_project(h, tower, grid_thw, B, out, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_merge_project(h, _ptr(tower), _grid(grid_thw), B, _ptr(out), _ptr(ws), ws_bytes,
                                _stream(stream)), "vt_merge_project")


def vt_attention_workspace_bytes(B, H, N, D) -> int:
    out = _sz()
    _check(lib.vt_attention_workspace_bytes(B, H, N, D, ctypes.byref(out)), "vt_attention_workspace_bytes")
    return out.value


def vt_attention(q, k, v, o, B, H, N, D, pos_thw, sections, theta, scale, ws, ws_bytes, stream=None) -> None:
    sec = (ctypes.c_int32 * 3)(*sections) if sections is not None else None
    _check(lib.vt_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, _ptr(pos_thw), sec, theta, scale,
                            _ptr(ws), ws_bytes, _stream(stream)), "vt_attention")


def vt_attention_static(q, k, v, o, B, H, N, D, pos_thw, sections, theta, scale, stream=None) -> None:
    """vt_attention without a workspace, for callers that cannot allocate device
    memory: its scratch is a fixed array inside the library (see include/vt.h)."""
    sec = (ctypes.c_int32 * 3)(*sections) if sections is not None else None
    _check(lib.vt_attention_static(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, D, _ptr(pos_thw), sec, theta,
                                   scale, _stream(stream)), "vt_attention_static")


def vt_attention_static_max_bytes() -> int:
    out = _sz()
    _check(lib.vt_attention_static_max_bytes(ctypes.byref(out)), "vt_attention_static_max_bytes")
    return out.value


def vt_attention_prepared(q, k, vt, ld_vt, o, B, H, N, D, scale, stream=None) -> None:
    _check(lib.vt_attention_prepared(_ptr(q), _ptr(k), _ptr(vt), ld_vt, _ptr(o), B, H, N, D, scale,
                                     _stream(stream)), "vt_attention_prepared")


def vt_linear(A, W, bias, resid, out, M, N, K, act=0, stream=None) -> None:
    _check(lib.vt_linear(_ptr(A), _ptr(W), _ptr(bias), _ptr(resid), _ptr(out), M, N, K, act, _stream(stream)),
           "vt_linear")


def vt_linear_ws(A, W, bias, resid, out, M, N, K, act, ws, ws_bytes, stream=None) -> None:
    _check(lib.vt_linear_ws(_ptr(A), _ptr(W), _ptr(bias), _ptr(resid), _ptr(out), M, N, K, act, _ptr(ws), ws_bytes,
                            _stream(stream)), "vt_linear_ws")


def vt_linear_workspace_bytes() -> int:
    n = _sz()
    _check(lib.vt_linear_workspace_bytes(ctypes.byref(n)), "vt_linear_workspace_bytes")
    return n.value


def vt_layernorm(x, gamma, beta, y, rows, cols, eps, stream=None) -> None:
    _check(lib.vt_layernorm(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(y), rows, cols, eps, _stream(stream)),
           "vt_layernorm")


def vt_patch_unfold(pixels, out, B, H, W, patch, temporal_patch, order, stream=None) -> None:
    _check(lib.vt_patch_unfold(_ptr(pixels), _ptr(out), B, H, W, patch, temporal_patch, order, _stream(stream)),
           "vt_patch_unfold")


def vt_index_maps(grid_thw):
    """Host-only: (token_order [N], pos_thw [N, 3], merge_src [N/4, 4]) as lists of ints."""
    t, h, w = (int(v) for v in grid_thw)
    n = t * h * w
    order = (ctypes.c_int32 * n)()
    pos = (ctypes.c_int32 * (3 * n))()
    merge = (ctypes.c_int32 * n)()
    _check(lib.vt_index_maps(_grid(grid_thw), order, pos, merge), "vt_index_maps")
    return list(order), [tuple(pos[3 * i:3 * i + 3]) for i in range(n)], \
        [tuple(merge[4 * i:4 * i + 4]) for i in range(n // 4)]


def vt_check(stream=None) -> None:
    _check(lib.vt_check(_stream(stream)), "vt_check")


def vt_selftest_wait_timeout(stream=None) -> None:
    _check(lib.vt_selftest_wait_timeout(_stream(stream)), "vt_selftest_wait_timeout")


def vt_profile_begin(stream=None) -> None:
    _check(lib.vt_profile_begin(_stream(stream)), "vt_profile_begin")


def vt_profile_end(stream=None) -> None:
    _check(lib.vt_profile_end(_stream(stream)), "vt_profile_end")


def vt_profile_read() -> dict:
    out = {}
    for cls, name in enumerate(PROFILE_CLASSES):
        ms, n = ctypes.c_double(), ctypes.c_int64()
        fl, by = ctypes.c_double(), ctypes.c_double()
        _check(lib.vt_profile_read(cls, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(fl), ctypes.byref(by)),
               "vt_profile_read")
        out[name] = dict(ms=ms.value, launches=n.value, flops=fl.value, bytes=by.value)
    return out


def vt_profile_launches() -> list[dict]:
    """Every launch of the last profiled interval: class name, ms, flops, bytes."""
    n = ctypes.c_int64()
    _check(lib.vt_profile_launches(ctypes.byref(n)), "vt_profile_launches")
    out = []
    for i in range(n.value):
        c, ms, fl, by = _i(), ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
        _check(lib.vt_profile_launch(i, ctypes.byref(c), ctypes.byref(ms), ctypes.byref(fl), ctypes.byref(by)),
               "vt_profile_launch")
        out.append(dict(cls=PROFILE_CLASSES[c.value], ms=ms.value, flops=fl.value, bytes=by.value))
    return out


# ------------------------------------------------------- model convenience

class Tower:
    """Owns a handle plus the device weights and workspace of one configuration."""

    def __init__(self, cfg: dict, weights_bits: dict, device="cuda"):
        import numpy as np
        import torch
        self.cfg = cfg
        self.h = vt_create(cfg)
        self.weights = {}
        for name, bits in weights_bits.items():
            t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
            self.weights[name] = t.to(device)
        vt_load_weights(self.h, self.weights)
        self._ws = None

    def workspace(self, B, grid_thw):
        import torch
        need = vt_workspace_bytes(self.h, B, grid_thw)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        return self._ws

    def close(self):
        if self.h:
            vt_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
