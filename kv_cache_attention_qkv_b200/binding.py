"""ctypes binding of libflashcache.so (include/flashcache.h).

Argument marshalling only: every step of the Flash-Cache path runs in the CUDA
library.  Tensors are torch CUDA tensors; the binding checks dtype, device and
contiguity (which the C ABI cannot see), passes raw pointers and the current
torch stream, and turns a non-zero status into ``FlashCacheError``.  If the
library is missing this module raises on import: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libflashcache.so")

FC_DTYPE_BF16 = 0
FC_DTYPE_FP32 = 1
STATUS = {0: "FC_OK", -1: "FC_ERR_INVALID_ARG", -2: "FC_ERR_UNSUPPORTED", -3: "FC_ERR_CUDA",
          -4: "FC_ERR_OOM", -5: "FC_ERR_DEVICE_CHECK", -6: "FC_ERR_TIMEOUT"}
DEVERR = {0x01: "POS_RANGE", 0x02: "POS_DUP", 0x04: "SEQLENS", 0x08: "CAND", 0x10: "TIMEOUT"}
EXPORTED = ("fc_create", "fc_step", "fc_topk_tracked", "fc_step_host", "fc_host_sync",
            "fc_get_error", "fc_last_launch_count", "fc_profile", "fc_profile_read",
            "fc_attention_noalloc", "fc_selftest_wait_timeout", "fc_destroy", "fc_status_str",
            "fc_model_create", "fc_model_step", "fc_model_layer_handle", "fc_model_destroy",
            "fc_decode_iteration", "fc_model_lm_head", "fc_last_step_work",
            "fc_last_cuda_error", "fc_profile_timeline", "fc_set_option", "fc_qkv_plan")
PROFILE_SLOTS = ("prep", "qkv_rope_scatter", "attention", "importance_finalize", "topk",
                 "attention_one_pass", "h2d_copy", "d2h_copy", "attention_split_pass1")


class FlashCacheError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class FcConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("rope_theta", ctypes.c_double), ("dtype", ctypes.c_int),
                ("max_batch", ctypes.c_int), ("max_total_q", ctypes.c_int),
                ("max_total_k", ctypes.c_int), ("max_seqlen_q", ctypes.c_int),
                ("max_pos", ctypes.c_int), ("max_topk", ctypes.c_int)]


class FcModelConfig(ctypes.Structure):
    _fields_ = [("layer", FcConfig), ("n_layers", ctypes.c_int), ("intermediate", ctypes.c_int),
                ("vocab", ctypes.c_int), ("max_head_rows", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("threshold", ctypes.c_float)]


class FcLayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gate", "w_up", "w_down")]


LAYER_WEIGHT_NAMES = tuple(n for n, _ in FcLayerWeights._fields_)

_lib = None


def load_library(path: Optional[str] = None):
    """Load libflashcache.so once and declare its signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FlashCacheError(-3, f"{p} is not built (run python -m kv_cache_attention_qkv_b200.build)")
    lib = ctypes.CDLL(p)
    vp, i32p, c_int = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_int
    lib.fc_create.argtypes = [ctypes.POINTER(FcConfig), vp, ctypes.POINTER(vp)]
    lib.fc_create.restype = c_int
    lib.fc_step.argtypes = [vp, vp, c_int, vp, vp, vp, vp, c_int, c_int, vp, vp, vp, vp, c_int]
    lib.fc_step.restype = c_int
    lib.fc_topk_tracked.argtypes = [vp, vp, c_int, c_int, vp, vp, vp, vp, vp, c_int, vp]
    lib.fc_topk_tracked.restype = c_int
    lib.fc_step_host.argtypes = [vp, vp, c_int, vp, vp, vp, vp, c_int, c_int, vp, vp, vp, vp, vp,
                                 c_int, vp, vp]
    lib.fc_step_host.restype = c_int
    lib.fc_host_sync.argtypes = [vp, vp]
    lib.fc_host_sync.restype = c_int
    lib.fc_qkv_plan.argtypes = [vp, c_int, i32p, i32p, i32p]
    lib.fc_qkv_plan.restype = c_int
    lib.fc_set_option.argtypes = [vp, c_int, c_int]
    lib.fc_set_option.restype = c_int
    lib.fc_last_cuda_error.argtypes = [vp]
    lib.fc_last_cuda_error.restype = ctypes.c_char_p
    lib.fc_last_step_work.argtypes = [vp, i32p, i32p, i32p]
    lib.fc_last_step_work.restype = c_int
    lib.fc_get_error.argtypes = [vp, i32p]
    lib.fc_get_error.restype = c_int
    lib.fc_last_launch_count.argtypes = [vp]
    lib.fc_last_launch_count.restype = c_int
    lib.fc_profile.argtypes = [vp, c_int]
    lib.fc_profile.restype = c_int
    lib.fc_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(c_int)]
    lib.fc_profile_timeline.argtypes = [vp, c_int, i32p, ctypes.POINTER(ctypes.c_float),
                                        ctypes.POINTER(ctypes.c_float), ctypes.POINTER(c_int)]
    lib.fc_profile_timeline.restype = c_int
    lib.fc_profile_read.restype = c_int
    lib.fc_selftest_wait_timeout.argtypes = [vp, vp, c_int]
    lib.fc_selftest_wait_timeout.restype = c_int
    lib.fc_attention_noalloc.argtypes = [vp, c_int, c_int, c_int, c_int, vp, vp, vp, c_int, c_int,
                                         vp, vp, vp, vp]
    lib.fc_attention_noalloc.restype = c_int
    lib.fc_destroy.argtypes = [vp]
    lib.fc_destroy.restype = None
    lib.fc_model_create.argtypes = [ctypes.POINTER(FcModelConfig), ctypes.POINTER(FcLayerWeights),
                                    vp, vp, ctypes.POINTER(vp)]
    lib.fc_model_create.restype = c_int
    lib.fc_model_step.argtypes = [vp, vp, c_int, vp, vp, vp, vp, c_int, c_int, vp, vp, vp, c_int,
                                  vp, vp, vp, vp, vp]
    lib.fc_model_step.restype = c_int
    lib.fc_model_layer_handle.argtypes = [vp]
    lib.fc_model_layer_handle.restype = vp
    lib.fc_model_destroy.argtypes = [vp]
    lib.fc_model_destroy.restype = None
    lib.fc_decode_iteration.argtypes = [vp, vp, c_int, vp, c_int, vp, vp, vp, c_int, c_int, c_int,
                                        vp, vp, vp, vp, vp, vp, vp]
    lib.fc_decode_iteration.restype = c_int
    lib.fc_model_lm_head.argtypes = [vp, vp, vp, c_int, vp, vp, vp]
    lib.fc_model_lm_head.restype = c_int
    lib.fc_status_str.argtypes = [c_int]
    lib.fc_status_str.restype = ctypes.c_char_p
    if path is None:
        _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class FlashCache:
    """One Flash-Cache layer: W_qkv bound at construction, steps on demand."""

    def __init__(self, w_qkv: torch.Tensor, *, hidden: int, n_heads: int, head_dim: int,
                 rope_theta: float, max_batch: int, max_total_q: int, max_total_k: int,
                 max_seqlen_q: int, max_pos: int, max_topk: int):
        self.lib = load_library()
        if w_qkv.dtype == torch.bfloat16:
            self.dtype, dt = torch.bfloat16, FC_DTYPE_BF16
        elif w_qkv.dtype == torch.float32:
            self.dtype, dt = torch.float32, FC_DTYPE_FP32
        else:
            raise FlashCacheError(-1, f"w_qkv dtype {w_qkv.dtype} is neither bfloat16 nor float32")
        if not (w_qkv.is_cuda and w_qkv.is_contiguous()):
            raise FlashCacheError(-1, "w_qkv must be a contiguous CUDA tensor")
        if tuple(w_qkv.shape) != (3 * n_heads * head_dim, hidden):
            raise FlashCacheError(-1, f"w_qkv shape {tuple(w_qkv.shape)} != [3*H*d, hidden]")
        self.w_qkv = w_qkv  # the library keeps the pointer: keep the tensor alive
        self.hidden, self.n_heads, self.head_dim = hidden, n_heads, head_dim
        self.cfg = FcConfig(hidden, n_heads, head_dim, float(rope_theta), dt, max_batch,
                            max_total_q, max_total_k, max_seqlen_q, max_pos, max_topk)
        self.device = w_qkv.device
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            st = self.lib.fc_create(ctypes.byref(self.cfg), _ptr(w_qkv), ctypes.byref(h))
        if st != 0:
            raise FlashCacheError(st, "fc_create")
        self._h = h

    # ------------------------------------------------------------------ checks
    def _check(self, t: torch.Tensor, name: str, dtype, ndim: Optional[int] = None):
        if t.dtype != dtype or not t.is_cuda or t.device != self.device or not t.is_contiguous():
            raise FlashCacheError(-1, f"{name}: need a contiguous {dtype} tensor on {self.device}")
        if ndim is not None and t.dim() != ndim:
            raise FlashCacheError(-1, f"{name}: need {ndim} dimensions, got {t.dim()}")

    def step(self, x, q_pos, cu_seqlens_q, cu_seqlens_k, k_cache, v_cache, out,
             importance=None, accumulate: bool = False, stream=None) -> None:
        """Enqueue fc_step on ``stream`` (default: torch's current stream)."""
        H, d = self.n_heads, self.head_dim
        self._check(x, "x", self.dtype, 2)
        self._check(q_pos, "q_pos", torch.int32, 1)
        self._check(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
        self._check(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
        for n, t in (("k_cache", k_cache), ("v_cache", v_cache), ("out", out)):
            self._check(t, n, self.dtype, 3)
            if t.shape[1:] != (H, d):
                raise FlashCacheError(-1, f"{n}: trailing shape {tuple(t.shape[1:])} != ({H}, {d})")
        T, S = x.shape[0], k_cache.shape[0]
        B = cu_seqlens_q.shape[0] - 1
        if (x.shape[1] != self.hidden or q_pos.shape[0] != T or out.shape[0] != T
                or v_cache.shape[0] != S or cu_seqlens_k.shape[0] != B + 1):
            raise FlashCacheError(-1, "fc_step: inconsistent shapes")
        if importance is not None:
            self._check(importance, "importance", torch.float32, 1)
            if importance.shape[0] != S:
                raise FlashCacheError(-1, "importance must have one entry per cache row")
        st = self.lib.fc_step(self._h, _stream_handle(stream), B, _ptr(x), _ptr(q_pos),
                              _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), T, S, _ptr(k_cache),
                              _ptr(v_cache), _ptr(out), _ptr(importance), int(bool(accumulate)))
        if st != 0:
            what = "fc_step"
            if st == -3:
                what += " (" + self.lib.fc_last_cuda_error(self._h).decode() + ")"
            raise FlashCacheError(st, what)

    def topk_tracked(self, importance, cu_seqlens_k, cand_lo, cand_hi, k: int, tracked,
                     k_per_seq=None, stream=None) -> None:
        """Enqueue fc_topk_tracked; ``tracked`` is int32 [B, k]."""
        self._check(importance, "importance", torch.float32, 1)
        for n, t in (("cu_seqlens_k", cu_seqlens_k), ("cand_lo", cand_lo), ("cand_hi", cand_hi)):
            self._check(t, n, torch.int32, 1)
        B = cu_seqlens_k.shape[0] - 1
        if k_per_seq is not None:
            self._check(k_per_seq, "k_per_seq", torch.int32, 1)
        self._check(tracked, "tracked", torch.int32, 2)
        if tuple(tracked.shape) != (B, k) or cand_lo.shape[0] != B or cand_hi.shape[0] != B:
            raise FlashCacheError(-1, "fc_topk_tracked: inconsistent shapes")
        st = self.lib.fc_topk_tracked(self._h, _stream_handle(stream), B, importance.shape[0],
                                      _ptr(importance), _ptr(cu_seqlens_k), _ptr(cand_lo),
                                      _ptr(cand_hi), _ptr(k_per_seq), int(k), _ptr(tracked))
        if st != 0:
            raise FlashCacheError(st, "fc_topk_tracked")

    def _check_host(self, t: torch.Tensor, name: str, dtype, ndim: int):
        if t.dtype != dtype or t.is_cuda or not t.is_contiguous() or t.dim() != ndim:
            raise FlashCacheError(-1, f"{name}: need a contiguous {dtype} host tensor, {ndim}-D")

    def step_host(self, x, q_pos, cu_seqlens_q, cu_seqlens_k, k_cache, v_cache, cand_lo, cand_hi,
                  k: int, out, tracked, k_per_seq=None, stream=None) -> None:
        """Enqueue fc_step_host: host (ideally pinned) inputs and outputs, device
        KV cache.  Outputs are valid after host_sync() and a sync of ``stream``."""
        H, d = self.n_heads, self.head_dim
        self._check_host(x, "x", self.dtype, 2)
        for n, t in (("q_pos", q_pos), ("cu_seqlens_q", cu_seqlens_q),
                     ("cu_seqlens_k", cu_seqlens_k), ("cand_lo", cand_lo), ("cand_hi", cand_hi)):
            self._check_host(t, n, torch.int32, 1)
        if k_per_seq is not None:
            self._check_host(k_per_seq, "k_per_seq", torch.int32, 1)
        self._check_host(out, "out", self.dtype, 3)
        self._check_host(tracked, "tracked", torch.int32, 2)
        for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
            self._check(t, n, self.dtype, 3)
        T, S = x.shape[0], k_cache.shape[0]
        B = cu_seqlens_q.shape[0] - 1
        if (x.shape[1] != self.hidden or q_pos.shape[0] != T or tuple(out.shape) != (T, H, d)
                or v_cache.shape[0] != S or cu_seqlens_k.shape[0] != B + 1
                or tuple(tracked.shape) != (B, k) or cand_lo.shape[0] != B or cand_hi.shape[0] != B):
            raise FlashCacheError(-1, "fc_step_host: inconsistent shapes")
        st = self.lib.fc_step_host(self._h, _stream_handle(stream), B, _ptr(x), _ptr(q_pos),
                                   _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), T, S, _ptr(k_cache),
                                   _ptr(v_cache), _ptr(cand_lo), _ptr(cand_hi), _ptr(k_per_seq),
                                   int(k), _ptr(out), _ptr(tracked))
        if st != 0:
            raise FlashCacheError(st, "fc_step_host")

    def host_sync(self, stream=None) -> None:
        """Make ``stream`` wait for every copy queued by step_host (fc_host_sync)."""
        st = self.lib.fc_host_sync(self._h, _stream_handle(stream))
        if st != 0:
            raise FlashCacheError(st, "fc_host_sync")

    def get_error(self) -> int:
        """Wait for the last stream used and return (and clear) the device error word."""
        w = ctypes.c_int32(0)
        st = self.lib.fc_get_error(self._h, ctypes.byref(w))
        if st not in (0, -5, -6):
            raise FlashCacheError(st, "fc_get_error")
        return int(w.value)

    def set_qkv_kernel(self, which: str, split: int = 0) -> None:
        """Projection kernel of the tensor-core path: "auto", "pair" or "splitk";
        ``split`` forces the split-K cluster size (0: chosen by shape)."""
        for opt, val in ((1, {"auto": 0, "pair": 1, "splitk": 2}[which]), (2, int(split))):
            st = self.lib.fc_set_option(self._h, opt, val)
            if st != 0:
                raise FlashCacheError(st, "fc_set_option")

    def set_attn_split(self, mode) -> None:
        """Small-batch attention split: True/"auto" (default: small batches with
        long caches), False/"never", or "always" (any cache length)."""
        val = {True: 0, "auto": 0, False: 1, "never": 1, "always": 2}[mode]
        st = self.lib.fc_set_option(self._h, 3, val)
        if st != 0:
            raise FlashCacheError(st, "fc_set_option")

    def qkv_plan(self, total_q: int) -> dict:
        """The projection kernel fc_step launches for ``total_q`` query rows."""
        k, sp, mc = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        st = self.lib.fc_qkv_plan(self._h, int(total_q), ctypes.byref(k), ctypes.byref(sp),
                                  ctypes.byref(mc))
        if st != 0:
            raise FlashCacheError(st, "fc_qkv_plan")
        return {"kernel": ("cuda_core", "pair", "splitk")[k.value], "split": sp.value,
                "max_clusters": mc.value}

    def last_step_work(self):
        """(work items, items of the two-pass kernel, items handed over to it) of
        the last step; waits for the last stream used."""
        a, b, c = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
        st = self.lib.fc_last_step_work(self._h, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
        if st != 0:
            raise FlashCacheError(st, "fc_last_step_work")
        return int(a.value), int(b.value), int(c.value)

    def profile(self, enable: bool) -> None:
        """Record a CUDA event pair around every later kernel launch (or stop)."""
        st = self.lib.fc_profile(self._h, int(bool(enable)))
        if st != 0:
            raise FlashCacheError(st, "fc_profile")

    def profile_read(self):
        """{kernel: (summed ms, launches)} since the last read; waits for the work."""
        ms = (ctypes.c_float * len(PROFILE_SLOTS))()
        n = (ctypes.c_int * len(PROFILE_SLOTS))()
        st = self.lib.fc_profile_read(self._h, ms, n)
        if st != 0:
            raise FlashCacheError(st, "fc_profile_read")
        return {name: (float(ms[i]), int(n[i])) for i, name in enumerate(PROFILE_SLOTS)}

    def profile_timeline(self, max_records: int = 4096):
        """[(kernel or copy slot, start ms, end ms)] of the records so far, times
        after the first record's start; call before profile_read (which clears)."""
        sl = (ctypes.c_int32 * max_records)()
        a = (ctypes.c_float * max_records)()
        b = (ctypes.c_float * max_records)()
        n = ctypes.c_int(0)
        st = self.lib.fc_profile_timeline(self._h, max_records, sl, a, b, ctypes.byref(n))
        if st != 0:
            raise FlashCacheError(st, "fc_profile_timeline")
        return [(PROFILE_SLOTS[sl[i]], float(a[i]), float(b[i])) for i in range(n.value)]

    def selftest_wait_timeout(self, limit_us: int, stream=None) -> None:
        """Enqueue the bounded-wait self-test (see fc_selftest_wait_timeout)."""
        st = self.lib.fc_selftest_wait_timeout(self._h, _stream_handle(stream), int(limit_us))
        if st != 0:
            raise FlashCacheError(st, "fc_selftest_wait_timeout")

    @property
    def last_launch_count(self) -> int:
        return int(self.lib.fc_last_launch_count(self._h))

    def close(self) -> None:
        if getattr(self, "_h", None):
            self.lib.fc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def describe_error_word(word: int):
    return [name for bit, name in DEVERR.items() if word & bit]


class FlashCacheModel:
    """The decoder stack around the Flash-Cache layer (fc_model_* of the C ABI):
    weights bound at construction, model steps on demand."""

    def __init__(self, layers, final_norm: torch.Tensor, lm_head: torch.Tensor, *, hidden: int,
                 n_heads: int, head_dim: int, rope_theta: float, intermediate: int, max_batch: int,
                 max_total_q: int, max_total_k: int, max_seqlen_q: int, max_pos: int,
                 max_topk: int, max_head_rows: int, rms_eps: float = 1e-5,
                 threshold: float = 0.9):
        self.lib = load_library()
        for t in [final_norm, lm_head] + [lw[n] for lw in layers for n in LAYER_WEIGHT_NAMES]:
            if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
                raise FlashCacheError(-1, "model weights must be contiguous bfloat16 CUDA tensors")
        self._keep = (layers, final_norm, lm_head)  # the library keeps the pointers
        self.n_layers, self.hidden = len(layers), hidden
        self.n_heads, self.head_dim = n_heads, head_dim
        self.device = lm_head.device
        cfg = FcModelConfig(FcConfig(hidden, n_heads, head_dim, float(rope_theta), FC_DTYPE_BF16,
                                     max_batch, max_total_q, max_total_k, max_seqlen_q, max_pos,
                                     max_topk),
                            len(layers), intermediate, lm_head.shape[0], max_head_rows,
                            float(rms_eps), float(threshold))
        arr = (FcLayerWeights * len(layers))()
        for i, lw in enumerate(layers):
            for n in LAYER_WEIGHT_NAMES:
                setattr(arr[i], n, lw[n].data_ptr())
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            st = self.lib.fc_model_create(ctypes.byref(cfg), arr, _ptr(final_norm), _ptr(lm_head),
                                          ctypes.byref(h))
        if st != 0:
            raise FlashCacheError(st, "fc_model_create")
        self._m = h

    def step(self, x, q_pos, cu_seqlens_q, cu_seqlens_k, k_caches, v_caches, head_rows=None,
             importance=None, token=None, confidence=None, accept=None, h_out=None,
             stream=None) -> None:
        """Enqueue fc_model_step; k_caches / v_caches are lists of [S, H, d] tensors."""
        if len(k_caches) != self.n_layers or len(v_caches) != self.n_layers:
            raise FlashCacheError(-1, "one K and one V cache per layer")
        T, S = x.shape[0], k_caches[0].shape[0]
        B = cu_seqlens_q.shape[0] - 1
        kp = (ctypes.c_void_p * self.n_layers)(*[t.data_ptr() for t in k_caches])
        vp_ = (ctypes.c_void_p * self.n_layers)(*[t.data_ptr() for t in v_caches])
        R = 0 if head_rows is None else head_rows.shape[0]
        st = self.lib.fc_model_step(self._m, _stream_handle(stream), B, _ptr(x), _ptr(q_pos),
                                    _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), T, S, kp, vp_,
                                    _ptr(head_rows), R, _ptr(importance), _ptr(token),
                                    _ptr(confidence), _ptr(accept), _ptr(h_out))
        if st != 0:
            raise FlashCacheError(st, "fc_model_step")

    def decode_iteration(self, cu_seqlens_k, k_caches, v_caches, embed, mask_id: int, tracked,
                         window_start, gen_end, tokens, draft, n_accepted, window: int,
                         importance=None, stream=None) -> None:
        """Enqueue fc_decode_iteration; tracked is int32 [B, K], the state arrays are
        int32 device tensors updated in place; importance (float [S] or None)
        receives the draft view's importance the reselection ranked."""
        if importance is not None and (importance.dtype != torch.float32 or not importance.is_cuda
                                       or not importance.is_contiguous()):
            raise FlashCacheError(-1, "importance must be a contiguous float32 CUDA tensor")
        B, K = tracked.shape
        kp = (ctypes.c_void_p * self.n_layers)(*[t.data_ptr() for t in k_caches])
        vp_ = (ctypes.c_void_p * self.n_layers)(*[t.data_ptr() for t in v_caches])
        st = self.lib.fc_decode_iteration(self._m, _stream_handle(stream), B, _ptr(cu_seqlens_k),
                                          k_caches[0].shape[0], kp, vp_, _ptr(embed), int(mask_id),
                                          int(K), int(window), _ptr(tracked), _ptr(window_start),
                                          _ptr(gen_end), _ptr(tokens), _ptr(draft),
                                          _ptr(n_accepted), _ptr(importance))
        if st != 0:
            raise FlashCacheError(st, "fc_decode_iteration")

    def lm_head(self, rows, token, confidence, accept, stream=None) -> None:
        """Enqueue fc_model_lm_head on final-normed bf16 rows [R, D]."""
        if rows.dtype != torch.bfloat16 or not rows.is_cuda or not rows.is_contiguous() or \
                rows.dim() != 2 or rows.shape[1] != self.hidden:
            raise FlashCacheError(-1, "rows must be a contiguous bfloat16 CUDA tensor [R, hidden]")
        R = rows.shape[0]
        for t, dt in ((token, torch.int32), (confidence, torch.float32), (accept, torch.uint8)):
            if t.dtype != dt or not t.is_cuda or not t.is_contiguous() or t.numel() < R:
                raise FlashCacheError(-1, "token/confidence/accept: int32/float32/uint8 CUDA [R]")
        st = self.lib.fc_model_lm_head(self._m, _stream_handle(stream), _ptr(rows), int(R),
                                       _ptr(token), _ptr(confidence), _ptr(accept))
        if st != 0:
            raise FlashCacheError(st, "fc_model_lm_head")

    def get_error(self) -> int:
        """Wait for the last stream used and return (and clear) the device error word."""
        w = ctypes.c_int32(0)
        st = self.lib.fc_get_error(self.lib.fc_model_layer_handle(self._m), ctypes.byref(w))
        if st not in (0, -5, -6):
            raise FlashCacheError(st, "fc_get_error")
        return int(w.value)

    @property
    def last_launch_count(self) -> int:
        return int(self.lib.fc_last_launch_count(self.lib.fc_model_layer_handle(self._m)))

    def close(self) -> None:
        if getattr(self, "_m", None):
            self.lib.fc_model_destroy(self._m)
            self._m = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
