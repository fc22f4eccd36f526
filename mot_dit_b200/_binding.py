"""ctypes binding of include/wam.h (argument marshalling only)."""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

FP32, BF16 = 0, 1
SEQUENTIAL, CEWP = 0, 1
PROF_CLASSES = ("video_norm", "video_qkv", "video_attn", "video_oproj", "video_ffn_up", "video_ffn_down",
                "video_temb", "video_io", "action_norm", "action_qkv", "action_attn", "action_oproj",
                "action_ffn_up", "action_ffn_down", "action_temb", "action_io", "action_block")

TRACE_KINDS = ("start", "video_kv", "video_end", "action_attn", "action_end", "end")

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
        "wam_infer_chunk_multistep": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, _F, C.c_int, _F, C.c_int, C.c_int, _P,
                                                _P]),
        "wam_tacd_targets": (C.c_int, [_P, _P, _P, _P, _P, _P, C.c_float, C.c_int, C.c_float] + [_P] * 6 + [_P]),
        "wam_export_params": (C.c_int, [_P, _P, C.POINTER(C.c_size_t)]),
        "wam_import_params": (C.c_int, [_P, _P, C.c_size_t]),
        "wam_read_kv": (C.c_int, [_P, C.c_int, C.c_int, _P, C.POINTER(C.c_size_t)]),
        "wam_check_device_status": (C.c_int, [_P]),
        "wam_chunk_kernel_count": (C.c_int, [_P, C.c_int]),
        "wam_profile_chunk": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, _P, _P, _P]),
        "wam_trace_chunk": (C.c_int, [_P, _P, _P, _P, _P, C.c_int, C.c_int, _P, _P, _P, C.c_int, _P]),
        "wam_test_peer_wait": (C.c_int, [C.c_int, C.c_uint64]),
        "wam_patchify": (C.c_int, [_P, _P] + [C.c_int] * 7 + [_P]),
        "wam_status_str": (C.c_char_p, [C.c_int]),
        "wam_last_error": (C.c_char_p, [_P]),
        "wam_op_linear": (C.c_int, [C.c_int, _P, _P, _P, _P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, _P]),
        "wam_op_linear_tiled": (C.c_int, [_P, _P, _P, _P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, _P]),
        "wam_op_attention_joint": (C.c_int, [_P, _P, _P, _P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                            C.c_int, _P]),
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


def _io(x, n: int, where: str, name: str, device: bool = True):
    """Pointer of a chunk I/O buffer after checking what the C ABI assumes of
    it: float32, C-contiguous, exactly n elements, in device memory (a CUDA
    tensor) for the device entry points or host memory (a numpy array or CPU
    tensor) for the host ones.  None and raw integer addresses pass through
    unchecked (the library rejects a missing required buffer)."""
    if x is None or isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        ok = not device and x.dtype == np.float32 and x.flags.c_contiguous and x.size == n
        got = f"numpy {x.dtype}, {x.size} elements"
    else:  # torch.Tensor
        ok = (bool(x.is_cuda) == device and str(x.dtype) == "torch.float32" and x.is_contiguous()
              and x.numel() == n)
        got = f"{'CUDA' if x.is_cuda else 'CPU'} tensor {x.dtype}, {x.numel()} elements"
    if not ok:
        where_mem = "device" if device else "host"
        raise WamError(1, where, f"{name}: need a C-contiguous float32 {where_mem} buffer of {n} elements, got {got}")
    return _ptr(x)


def _check_sched(t, S: int, where: str):
    if t is not None and len(t) != S + 1:
        raise WamError(1, where, f"t_sched has {len(t)} values, S + 1 = {S + 1} needed")


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

    def io_sizes(self):
        """Element counts of one chunk's (video, cond, actions) buffers:
        [B, l_video, d_video or video_patch_dim], [B, l_cond, d_video] and
        [B, l_action, action_dim]."""
        c = self.cfg
        return (c.batch * c.l_video * (c.video_patch_dim or c.d_video), c.batch * c.l_cond * c.d_video,
                c.batch * c.l_action * c.action_dim)

    def _chunk_ptrs(self, where, video, cond, noise, out, device=True):
        nv, nc, na = self.io_sizes()
        return (_io(video, nv, where, "video", device), _io(cond, nc, where, "cond", device),
                _io(noise, na, where, "noise", device), _io(out, na, where, "out", device))

    def video_forward(self, video, cond, t_video=0.0, stream=None):
        nv, nc, _ = self.io_sizes()
        w = "wam_video_forward"
        self._check(self._lib.wam_video_forward(self._h, _io(video, nv, w, "video"), _io(cond, nc, w, "cond"),
                                                t_video, _stream(stream)), w)

    def action_step(self, actions, t_from, t_to, stream=None):
        w = "wam_action_step"
        self._check(self._lib.wam_action_step(self._h, _io(actions, self.io_sizes()[2], w, "actions"), t_from, t_to,
                                              _stream(stream)), w)

    def infer_chunk(self, video, cond, noise, out, S=1, t_sched=None, mode=CEWP, use_graph=True,
                    stream_video=None, stream_action=None):
        w = "wam_infer_chunk"
        ptrs = self._chunk_ptrs(w, video, cond, noise, out)
        _check_sched(t_sched, S, w)
        p, keep = _sched(t_sched)
        self._check(self._lib.wam_infer_chunk(self._h, *ptrs, S, p, mode, int(use_graph), _stream(stream_video),
                                              _stream(stream_action)), w)
        del keep

    def infer_chunk_host(self, video, cond, noise, out, S=1, t_sched=None, mode=CEWP, use_graph=True,
                         stream_video=None, stream_action=None):
        w = "wam_infer_chunk_host"
        ptrs = self._chunk_ptrs(w, video, cond, noise, out, device=False)
        _check_sched(t_sched, S, w)
        p, keep = _sched(t_sched)
        self._check(self._lib.wam_infer_chunk_host(self._h, *ptrs, S, p, mode, int(use_graph),
                                                   _stream(stream_video), _stream(stream_action)), w)
        del keep

    def joint_one_step(self, video_clean, video_eps, action_clean, action_eps, u_video, u_action,
                       video_out, action_out, shift_video=5.0, shift_action=1.0, mode=CEWP, use_graph=True,
                       stream_video=None, stream_action=None):
        w = "wam_joint_one_step"
        nv, _, na = self.io_sizes()
        self._check(self._lib.wam_joint_one_step(
            self._h, _io(video_clean, nv, w, "video_clean"), _io(video_eps, nv, w, "video_eps"),
            _io(action_clean, na, w, "action_clean"), _io(action_eps, na, w, "action_eps"), u_video, u_action,
            shift_video, shift_action, _io(video_out, nv, w, "video_out"), _io(action_out, na, w, "action_out"),
            mode, int(use_graph), _stream(stream_video), _stream(stream_action)), w)

    def infer_chunk_multistep(self, video_eps, noise, video_out, actions_out, n_video=1, sched_video=None, S=1,
                              t_sched=None, mode=CEWP, use_graph=True, stream_video=None, stream_action=None):
        w = "wam_infer_chunk_multistep"
        nv, _, na = self.io_sizes()
        _check_sched(sched_video, n_video, w)
        _check_sched(t_sched, S, w)
        pv, keep_v = _sched(sched_video)
        pa, keep_a = _sched(t_sched)
        self._check(self._lib.wam_infer_chunk_multistep(
            self._h, _io(video_eps, nv, w, "video_eps"), _io(noise, na, w, "noise"), _io(video_out, nv, w, "video_out"),
            _io(actions_out, na, w, "actions_out"), n_video, pv, S, pa, mode, int(use_graph), _stream(stream_video),
            _stream(stream_action)), w)
        del keep_v, keep_a

    def tacd_targets(self, ema, video, cond, action_clean, eps, t, K, lam, u_ta, v_student, u_cd, losses,
                     a_t=None, a0_teacher=None, stream=None):
        """TACD target forward (wam_tacd_targets): this context is the student
        (its base weights are the teacher), `ema` the EMA target (may be self)."""
        w = "wam_tacd_targets"
        nv, nc, na = self.io_sizes()
        ema_h = ema._h if ema is not None else None
        self._check(self._lib.wam_tacd_targets(
            self._h, ema_h, _io(video, nv, w, "video"), _io(cond, nc, w, "cond"),
            _io(action_clean, na, w, "action_clean"), _io(eps, na, w, "eps"), t, K, lam,
            _io(u_ta, na, w, "u_ta"), _io(v_student, na, w, "v_student"), _io(u_cd, na, w, "u_cd"),
            _io(losses, 3, w, "losses"), _io(a_t, na, w, "a_t"), _io(a0_teacher, na, w, "a0_teacher"),
            _stream(stream)), w)

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

    def trace_chunk(self, video, cond, noise, out, S=1, mode=CEWP, stream_video=None, stream_action=None):
        """Block-boundary timestamps of one graph-replayed chunk: a list of
        (kind, block, step, ms) with kind in TRACE_KINDS."""
        w = "wam_trace_chunk"
        ptrs = self._chunk_ptrs(w, video, cond, noise, out)
        cap = 8 * (self.cfg.n_blocks + 2) * (S + 1)
        buf = np.zeros(4 * cap, np.float32)
        n = C.c_int(0)
        self._check(self._lib.wam_trace_chunk(self._h, *ptrs, S, mode, _stream(stream_video), _stream(stream_action),
                                              buf.ctypes.data, cap, C.byref(n)), w)
        rec = buf[:4 * min(n.value, cap)].reshape(-1, 4)
        return [(TRACE_KINDS[int(k)], int(b), int(j), float(t)) for k, b, j, t in rec]

    def profile_chunk(self, video, cond, noise, out, S=1, stream=None):
        """Per-class summed launch durations (ms) and launch counts of one eager
        sequential chunk (see PROF_CLASSES)."""
        ms = np.zeros(len(PROF_CLASSES), np.float32)
        cnt = np.zeros(len(PROF_CLASSES), np.int32)
        w = "wam_profile_chunk"
        ptrs = self._chunk_ptrs(w, video, cond, noise, out)
        self._check(self._lib.wam_profile_chunk(self._h, *ptrs, S, _stream(stream), ms.ctypes.data, cnt.ctypes.data),
                    w)
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(PROF_CLASSES)}


def op_linear(dtype, x, w, bias, out, M, N, K, swap=False, splits=1, stream=None):
    st = lib().wam_op_linear(dtype, _ptr(x), _ptr(w), _ptr(bias), _ptr(out), M, N, K, int(swap), splits,
                             _stream(stream))
    if st:
        raise WamError(st, "wam_op_linear")


def op_linear_tiled(x, w, bias, out, M, N, K, bn=256, mode=1, ctas=0, stream=None):
    """mode 0: single CTAs; 1: CTA pairs (2-SM MMA); 2: clusters of two, split tiles finished in halves;
    3: swapped (M <= 64 tokens), each tile split over a cluster of `ctas` CTAs summed in shared memory."""
    st = lib().wam_op_linear_tiled(_ptr(x), _ptr(w), _ptr(bias), _ptr(out), M, N, K, bn, int(mode), ctas,
                                   _stream(stream))
    if st:
        raise WamError(st, "wam_op_linear_tiled")


def op_attention_joint(q, k, v, out, B, H, Lq, Lk, Lcache, ready=0, splits=0, stream=None):
    st = lib().wam_op_attention_joint(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Lq, Lk, Lcache, ready, splits,
                                      _stream(stream))
    if st:
        raise WamError(st, "wam_op_attention_joint")


def op_norm_mod(dtype, x, h, M, d, scale=None, shift=None, gain=None, stream=None):
    st = lib().wam_op_norm_mod(dtype, _ptr(x), _ptr(h), M, d, _ptr(scale), _ptr(shift), _ptr(gain), _stream(stream))
    if st:
        raise WamError(st, "wam_op_norm_mod")


def op_attention(dtype, q, k, v, out, B, H, Dh, Lq, Lk, Lcache, splits=1, stream=None):
    st = lib().wam_op_attention(dtype, _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Dh, Lq, Lk, Lcache, splits,
                                _stream(stream))
    if st:
        raise WamError(st, "wam_op_attention")


def patchify(frames, patches, B, F, C, H, W, p, inverse=False, stream=None):
    """Frames [B, F, C, H, W] <-> patch tokens [B, F (H/p)(W/p), C p p] (wam_patchify)."""
    st = lib().wam_patchify(_ptr(frames), _ptr(patches), B, F, C, H, W, p, int(inverse), _stream(stream))
    if st:
        raise WamError(st, "wam_patchify")


def op_attention_noalloc(q, k, v, out, B, H, Lq, Lk, Lcache, splits, stream=None):
    """Split-KV bf16 attention with library-owned static scratch (no allocation)."""
    st = lib().wam_op_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Lq, Lk, Lcache, splits,
                                        _stream(stream))
    if st:
        raise WamError(st, "wam_op_attention_noalloc")
