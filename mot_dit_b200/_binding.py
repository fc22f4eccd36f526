"""ctypes binding of include/wam.h (argument marshalling only)."""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

FP32, BF16 = 0, 1
SEQUENTIAL, CEWP = 0, 1
PROF_CLASSES = ("video_norm", "video_qkv", "video_attn", "video_oproj", "video_ffn_up", "video_ffn_down",
                "video_temb", "video_io", "action_norm", "action_qkv", "action_attn", "action_oproj",
                "action_ffn_up", "action_ffn_down", "action_temb", "action_io")

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "out of device memory", 4: "CUDA error",
           5: "device wait timed out", 6: "invalid call order"}


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmotdit.so")


class WamError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class WamConfig(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "n_blocks", "d_video", "d_action", "n_heads", "head_dim", "ffn_video", "ffn_action",
        "l_cond", "l_video", "l_action", "action_dim", "video_patch_dim", "batch", "lora_rank")] + [
        ("lora_scale", C.c_float), ("video_has_output", C.c_int), ("dtype", C.c_int)]

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n, _ in self._fields_}

    def replace(self, **kw) -> "WamConfig":
        c = WamConfig(**self.as_dict())
        for k, v in kw.items():
            setattr(c, k, v)
        return c


_lib = None
_P = C.c_void_p
_F = C.POINTER(C.c_float)


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m mot_dit_b200.build` "
                           "(there is no fallback implementation)")
    L = C.CDLL(path)
    sig = {
        "wam_preset": (C.c_int, [C.c_int, C.POINTER(WamConfig)]),
        "wam_init": (C.c_int, [C.POINTER(WamConfig), C.c_uint64, C.POINTER(_P)]),
        "wam_destroy": (None, [_P]),
        "wam_video_forward": (C.c_int, [_P, _P, _P, C.c_float, _P]),
        "wam_action_step": (C.c_int, [_P, _P, C.c_float, C.c_float, _P]),
        "wam_infer_chunk": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, _F, C.c_int, C.c_int, _P, _P]),
        "wam_infer_chunk_host": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, _F, C.c_int, C.c_int, _P, _P]),
        "wam_joint_one_step": (C.c_int, [_P, _P, _P, _P, _P, C.c_float, C.c_float, C.c_float, C.c_float, _P, _P,
                                         C.c_int, C.c_int, _P, _P]),
        "wam_export_params": (C.c_int, [_P, _P, C.POINTER(C.c_size_t)]),
        "wam_import_params": (C.c_int, [_P, _P, C.c_size_t]),
        "wam_read_kv": (C.c_int, [_P, C.c_int, C.c_int, _P, C.POINTER(C.c_size_t)]),
        "wam_check_device_status": (C.c_int, [_P]),
        "wam_chunk_kernel_count": (C.c_int, [_P, C.c_int]),
        "wam_profile_chunk": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, _P, _P, _P]),
        "wam_status_str": (C.c_char_p, [C.c_int]),
        "wam_last_error": (C.c_char_p, [_P]),
        "wam_op_linear": (C.c_int, [C.c_int, _P, _P, _P, _P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, _P]),
        "wam_op_attention": (C.c_int, [C.c_int, _P, _P, _P, _P] + [C.c_int] * 7 + [_P]),
        "wam_op_attention_noalloc": (C.c_int, [_P, _P, _P, _P] + [C.c_int] * 6 + [_P]),
        "wam_op_norm_mod": (C.c_int, [C.c_int, _P, _P, C.c_int, C.c_int, _P, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def preset(k: int) -> WamConfig:
    c = WamConfig()
    st = lib().wam_preset(k, C.byref(c))
    if st:
        raise WamError(st, f"wam_preset({k})")
    return c


def _ptr(x):
    """Device/host pointer of a torch tensor, numpy array, int or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()  # torch.Tensor


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream  # torch.cuda.Stream


def _sched(t):
    if t is None:
        return None, None
    arr = (C.c_float * len(t))(*[float(v) for v in t])
    return C.cast(arr, _F), arr


class Wam:
    """One model context (seeded weights resident on the current device)."""

    def __init__(self, cfg, seed: int = 0):
        self.cfg = preset(cfg) if isinstance(cfg, int) else cfg
        self._lib = lib()
        h = _P()
        st = self._lib.wam_init(C.byref(self.cfg), C.c_uint64(seed), C.byref(h))
        if st:
            raise WamError(st, "wam_init")
        self._h = h

    def _check(self, st, where):
        if st:
            raise WamError(st, where, self._lib.wam_last_error(self._h).decode())

    def close(self):
        if getattr(self, "_h", None):
            self._lib.wam_destroy(self._h)
            self._h = None

    __del__ = close

    def video_forward(self, video, cond, t_video=0.0, stream=None):
        self._check(self._lib.wam_video_forward(self._h, _ptr(video), _ptr(cond), t_video, _stream(stream)),
                    "wam_video_forward")

    def action_step(self, actions, t_from, t_to, stream=None):
        self._check(self._lib.wam_action_step(self._h, _ptr(actions), t_from, t_to, _stream(stream)),
                    "wam_action_step")

    def infer_chunk(self, video, cond, noise, out, S=1, t_sched=None, mode=CEWP, use_graph=True,
                    stream_video=None, stream_action=None):
        p, keep = _sched(t_sched)
        self._check(self._lib.wam_infer_chunk(self._h, _ptr(video), _ptr(cond), _ptr(noise), _ptr(out), S, p,
                                              mode, int(use_graph), _stream(stream_video),
                                              _stream(stream_action)), "wam_infer_chunk")
        del keep

    def infer_chunk_host(self, video, cond, noise, out, S=1, t_sched=None, mode=CEWP, use_graph=True,
                         stream_video=None, stream_action=None):
        p, keep = _sched(t_sched)
        self._check(self._lib.wam_infer_chunk_host(self._h, _ptr(video), _ptr(cond), _ptr(noise), _ptr(out), S, p,
                                                   mode, int(use_graph), _stream(stream_video),
                                                   _stream(stream_action)), "wam_infer_chunk_host")
        del keep

    def joint_one_step(self, video_clean, video_eps, action_clean, action_eps, u_video, u_action,
                       video_out, action_out, shift_video=5.0, shift_action=1.0, mode=CEWP, use_graph=True,
                       stream_video=None, stream_action=None):
        self._check(self._lib.wam_joint_one_step(
            self._h, _ptr(video_clean), _ptr(video_eps), _ptr(action_clean), _ptr(action_eps), u_video, u_action,
            shift_video, shift_action, _ptr(video_out), _ptr(action_out), mode, int(use_graph),
            _stream(stream_video), _stream(stream_action)), "wam_joint_one_step")

    def export_params(self) -> np.ndarray:
        n = C.c_size_t(0)
        self._check(self._lib.wam_export_params(self._h, None, C.byref(n)), "wam_export_params")
        out = np.empty(n.value // 4, np.float32)
        self._check(self._lib.wam_export_params(self._h, out.ctypes.data, C.byref(n)), "wam_export_params")
        return out

    def import_params(self, flat: np.ndarray):
        flat = np.ascontiguousarray(flat, dtype=np.float32)
        self._check(self._lib.wam_import_params(self._h, flat.ctypes.data, flat.nbytes), "wam_import_params")

    def read_kv(self, block: int, which: int) -> np.ndarray:
        n = C.c_size_t(0)
        self._check(self._lib.wam_read_kv(self._h, block, which, None, C.byref(n)), "wam_read_kv")
        out = np.empty(n.value // 4, np.float32)
        self._check(self._lib.wam_read_kv(self._h, block, which, out.ctypes.data, C.byref(n)), "wam_read_kv")
        c = self.cfg
        return out.reshape(c.batch, c.n_heads, c.l_cond + c.l_video + c.l_action, c.head_dim)

    def check_device_status(self):
        self._check(self._lib.wam_check_device_status(self._h), "wam_check_device_status")

    def chunk_kernel_count(self, S: int) -> int:
        return self._lib.wam_chunk_kernel_count(self._h, S)

    def profile_chunk(self, video, cond, noise, out, S=1, stream=None):
        """Per-class summed launch durations (ms) and launch counts of one eager
        sequential chunk (see PROF_CLASSES)."""
        ms = np.zeros(len(PROF_CLASSES), np.float32)
        cnt = np.zeros(len(PROF_CLASSES), np.int32)
        self._check(self._lib.wam_profile_chunk(self._h, _ptr(video), _ptr(cond), _ptr(noise), _ptr(out), S,
                                                _stream(stream), ms.ctypes.data, cnt.ctypes.data),
                    "wam_profile_chunk")
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(PROF_CLASSES)}


def op_linear(dtype, x, w, bias, out, M, N, K, swap=False, splits=1, stream=None):
    st = lib().wam_op_linear(dtype, _ptr(x), _ptr(w), _ptr(bias), _ptr(out), M, N, K, int(swap), splits,
                             _stream(stream))
    if st:
        raise WamError(st, "wam_op_linear")


def op_norm_mod(dtype, x, h, M, d, scale=None, shift=None, gain=None, stream=None):
    st = lib().wam_op_norm_mod(dtype, _ptr(x), _ptr(h), M, d, _ptr(scale), _ptr(shift), _ptr(gain), _stream(stream))
    if st:
        raise WamError(st, "wam_op_norm_mod")


def op_attention(dtype, q, k, v, out, B, H, Dh, Lq, Lk, Lcache, splits=1, stream=None):
    st = lib().wam_op_attention(dtype, _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Dh, Lq, Lk, Lcache, splits,
                                _stream(stream))
    if st:
        raise WamError(st, "wam_op_attention")


def op_attention_noalloc(q, k, v, out, B, H, Lq, Lk, Lcache, splits, stream=None):
    """Split-KV bf16 attention with library-owned static scratch (no allocation)."""
    st = lib().wam_op_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Lq, Lk, Lcache, splits,
                                        _stream(stream))
    if st:
        raise WamError(st, "wam_op_attention_noalloc")
