"""ctypes binding of the C ABI in ``include/pa.h``.

Argument marshalling only: tensors are checked for dtype, shape, device and
contiguity, then their device pointers and the current CUDA stream are passed
to ``libpa_b200.so``.  Every step of the attention runs in the library's
kernels; there is no other implementation behind this module, and it raises if
the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpa_b200.so")

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA = 0, 1, 2, 3
STATUS_BAD_PAGE = 1 << 0
STATUS_Q_GT_KV = 1 << 1
STATUS_KV_GT_CAPACITY = 1 << 2
STATUS_BAD_CU_Q = 1 << 3
STATUS_TIMEOUT = 1 << 4

EXPORTS = ("pa_create_plan", "pa_run", "pa_destroy", "pa_last_error", "pa_set_scale",
           "pa_set_num_pages", "pa_set_num_splits", "pa_get_status", "pa_workspace_bytes",
           "pa_max_splits", "pa_profile_start", "pa_profile_read", "pa_run_noalloc",
           "pa_set_two_stage_prefill", "pa_set_decode_kernel", "pa_append_kv",
           "pa_set_causal", "pa_set_page_table_stride", "pa_set_fused_merge", "pa_set_kv_fp8",
           "pa_selftest_wait_timeout", "pa_noalloc_get_status", "pa_set_kv_fp8_widen")

# Size of the library's static scratch array used by pa_run_noalloc.
NOALLOC_SCRATCH_BYTES = 8 << 20

_lib = None


class PAError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("%s (code %d)" % (msg, code))
        self.code = code


def load_library(path: str = LIB_PATH):
    """Load ``libpa_b200.so`` and declare the C signatures."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("paged_kv_gqa_fmha_b200: CUDA library %s is missing; build it with "
                           "`python -m paged_kv_gqa_fmha_b200._build`" % path)
    lib = ctypes.CDLL(path)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.pa_create_plan.argtypes = [I, I, I, I, I, I]
    lib.pa_create_plan.restype = P
    lib.pa_run.argtypes = [P, P, P, P, P, P, P, P, P, P]
    lib.pa_run.restype = I
    lib.pa_destroy.argtypes = [P]
    lib.pa_destroy.restype = None
    lib.pa_last_error.argtypes = []
    lib.pa_last_error.restype = ctypes.c_char_p
    lib.pa_set_scale.argtypes = [P, F]
    lib.pa_set_scale.restype = I
    lib.pa_set_num_pages.argtypes = [P, I]
    lib.pa_set_num_pages.restype = I
    lib.pa_set_num_splits.argtypes = [P, I]
    lib.pa_set_num_splits.restype = I
    lib.pa_get_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32), I]
    lib.pa_get_status.restype = I
    lib.pa_workspace_bytes.argtypes = [P]
    lib.pa_workspace_bytes.restype = ctypes.c_size_t
    lib.pa_max_splits.argtypes = [P]
    lib.pa_max_splits.restype = I
    lib.pa_profile_start.argtypes = [P, I]
    lib.pa_profile_start.restype = I
    lib.pa_profile_read.argtypes = [P, ctypes.POINTER(F), ctypes.POINTER(I), ctypes.POINTER(I)]
    lib.pa_profile_read.restype = I
    lib.pa_set_two_stage_prefill.argtypes = [P, I]
    lib.pa_set_two_stage_prefill.restype = I
    lib.pa_set_decode_kernel.argtypes = [P, I]
    lib.pa_set_decode_kernel.restype = I
    lib.pa_append_kv.argtypes = [P, P, P, P, P, P, P, P, P]
    lib.pa_append_kv.restype = I
    lib.pa_set_causal.argtypes = [P, I]
    lib.pa_set_causal.restype = I
    lib.pa_set_fused_merge.argtypes = [P, I]
    lib.pa_set_fused_merge.restype = I
    lib.pa_set_page_table_stride.argtypes = [P, I]
    lib.pa_set_page_table_stride.restype = I
    lib.pa_set_kv_fp8.argtypes = [P, I, F, F]
    lib.pa_set_kv_fp8.restype = I
    lib.pa_set_kv_fp8_widen.argtypes = [P, I]
    lib.pa_set_kv_fp8_widen.restype = I
    lib.pa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint32),
                                             ctypes.POINTER(ctypes.c_uint32)]
    lib.pa_selftest_wait_timeout.restype = I
    lib.pa_run_noalloc.argtypes = [I, I, I, I, I, I, I, F, P, P, P, P, P, P, P, P, P]
    lib.pa_run_noalloc.restype = I
    lib.pa_noalloc_get_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), I]
    lib.pa_noalloc_get_status.restype = I
    if path == LIB_PATH:
        _lib = lib
    return lib


def last_error() -> str:
    return load_library().pa_last_error().decode()


def _check(rc):
    if rc != PA_OK:
        raise PAError(rc, last_error())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class Plan:
    """One geometry (batch, heads, head_dim, page size, capacity): owns the
    device workspace; ``run`` binds the request metadata of each call."""

    def __init__(self, batch, heads_q, heads_kv, head_dim, page_size, capacity,
                 scale: Optional[float] = None, num_pages: int = 0, num_splits: int = 0):
        self._lib = load_library()
        self._h = self._lib.pa_create_plan(batch, heads_q, heads_kv, head_dim, page_size,
                                           capacity)
        if not self._h:
            raise PAError(PA_ERR_INVALID, last_error())
        self.batch, self.heads_q, self.heads_kv = batch, heads_q, heads_kv
        self.head_dim, self.page_size, self.capacity = head_dim, page_size, capacity
        self._tstride = capacity
        self._kv_dtype = torch.bfloat16
        if scale is not None:
            _check(self._lib.pa_set_scale(self._h, float(scale)))
        if num_pages:
            _check(self._lib.pa_set_num_pages(self._h, int(num_pages)))
        if num_splits:
            _check(self._lib.pa_set_num_splits(self._h, int(num_splits)))

    def set_num_pages(self, n: int):
        _check(self._lib.pa_set_num_pages(self._h, int(n)))

    def set_num_splits(self, n: int):
        _check(self._lib.pa_set_num_splits(self._h, int(n)))

    def set_two_stage_prefill(self, on: bool):
        _check(self._lib.pa_set_two_stage_prefill(self._h, 1 if on else 0))

    def set_decode_kernel(self, on: bool):
        """Decode-only runs (cu_q_lens None): True puts head_dim 128 and 256 on
        the keys-as-M decode kernel, False puts both on the one-stage kernel
        (default: head_dim 128 on the decode kernel, 256 on the one-stage)."""
        _check(self._lib.pa_set_decode_kernel(self._h, 1 if on else 0))

    def set_fused_merge(self, on: bool):
        """True: split-KV partials are merged by the last split warp of each
        (request, KV head); False (default): by a separate merge kernel."""
        _check(self._lib.pa_set_fused_merge(self._h, 1 if on else 0))

    def set_kv_fp8(self, on: bool, k_scale: float = 1.0, v_scale: float = 1.0):
        """True: the pools of later ``run`` calls are uint8 tensors of E4M3
        codes, read as ``k_scale * code`` and ``v_scale * code`` (decode runs,
        prefill and mixed batches).  False: bf16 pools."""
        _check(self._lib.pa_set_kv_fp8(self._h, 1 if on else 0, float(k_scale), float(v_scale)))
        self._kv_dtype = torch.uint8 if on else torch.bfloat16

    def set_kv_fp8_widen(self, max_pages: int):
        """Scratch capacity in pages for E4M3 requests of two or more query
        blocks, which are widened once per run and read as bf16 pages
        (-1 automatic, 0 never)."""
        _check(self._lib.pa_set_kv_fp8_widen(self._h, int(max_pages)))

    def set_causal(self, causal: bool):
        """True (default): causal mask aligned to the end of KV; False: every
        query row sees all of its request's keys."""
        _check(self._lib.pa_set_causal(self._h, 1 if causal else 0))

    def _bind_table(self, page_table):
        """Accept a [B, C] int32 table whose rows may be strided (e.g. the K
        plane of a [B, 2, C] tensor, row stride 2C) and pass its stride on."""
        B = self.batch
        if (page_table.dtype != torch.int32 or page_table.dim() != 2
                or tuple(page_table.shape) != (B, self.capacity) or page_table.stride(1) != 1
                or page_table.stride(0) < self.capacity):
            raise ValueError("page_table must be an int32 [%d, %d] tensor with unit column "
                             "stride and row stride >= %d" % (B, self.capacity, self.capacity))
        if page_table.stride(0) != self._tstride:
            _check(self._lib.pa_set_page_table_stride(self._h, int(page_table.stride(0))))
            self._tstride = int(page_table.stride(0))

    def set_scale(self, s: float):
        _check(self._lib.pa_set_scale(self._h, float(s)))

    @property
    def workspace_bytes(self) -> int:
        return int(self._lib.pa_workspace_bytes(self._h))

    @property
    def max_splits(self) -> int:
        return int(self._lib.pa_max_splits(self._h))

    def run(self, q, k_pool, v_pool, page_table, seq_lens, cu_q_lens=None, out=None, lse=None,
            want_lse=True, stream=None):
        """Enqueue one pass on ``stream`` (default: torch's current stream).
        Returns (out, lse); lse is None if ``want_lse`` is False and no ``lse``
        tensor was given."""
        B, Hq, Hkv, D = self.batch, self.heads_q, self.heads_kv, self.head_dim
        dev = q.device
        if dev.type != "cuda":
            raise ValueError("tensors must be on a CUDA device")
        for name, t, dt in (("q", q, torch.bfloat16), ("k_pool", k_pool, self._kv_dtype),
                            ("v_pool", v_pool, self._kv_dtype),
                            ("seq_lens", seq_lens, torch.int32)):
            if t.dtype != dt or t.device != dev or not t.is_contiguous():
                raise ValueError("%s must be a contiguous %s tensor on %s" % (name, dt, dev))
        if page_table.device != dev:
            raise ValueError("page_table must be on %s" % dev)
        self._bind_table(page_table)
        if q.dim() != 3 or q.shape[1] != Hq or q.shape[2] != D:
            raise ValueError("q must be [T, %d, %d], got %s" % (Hq, D, tuple(q.shape)))
        if k_pool.dim() != 4 or tuple(k_pool.shape[1:]) != (self.page_size, Hkv, D):
            raise ValueError("k_pool must be [P, %d, %d, %d], got %s"
                             % (self.page_size, Hkv, D, tuple(k_pool.shape)))
        if v_pool.shape != k_pool.shape:
            raise ValueError("v_pool shape %s != k_pool shape %s"
                             % (tuple(v_pool.shape), tuple(k_pool.shape)))
        if tuple(seq_lens.shape) != (B,):
            raise ValueError("seq_lens must be [%d]" % B)
        if cu_q_lens is not None:
            if (cu_q_lens.dtype != torch.int32 or tuple(cu_q_lens.shape) != (B + 1,)
                    or cu_q_lens.device != dev or not cu_q_lens.is_contiguous()):
                raise ValueError("cu_q_lens must be a contiguous int32 [%d] tensor" % (B + 1))
        elif q.shape[0] != B:
            raise ValueError("without cu_q_lens, q must hold one token per request")
        T = q.shape[0]
        if out is None:
            out = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=dev)
        if lse is None and want_lse:
            lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
        if stream is None:
            stream = torch.cuda.current_stream(dev).cuda_stream
        elif isinstance(stream, torch.cuda.Stream):
            stream = stream.cuda_stream
        _check(self._lib.pa_run(self._h, _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table),
                                _ptr(seq_lens), _ptr(cu_q_lens), _ptr(out), _ptr(lse),
                                ctypes.c_void_p(stream)))
        return out, lse

    def append_kv(self, k_new, v_new, k_pool, v_pool, page_table, seq_lens, cu_q_lens=None,
                  stream=None):
        """Write this step's new K/V rows ([T, Hkv, D] bf16, packed like q) into
        the pools in place (``pa_append_kv``); stream-ordered."""
        B, Hkv, D = self.batch, self.heads_kv, self.head_dim
        dev = k_new.device
        if dev.type != "cuda":
            raise ValueError("tensors must be on a CUDA device")
        for name, t, dt in (("k_new", k_new, torch.bfloat16), ("v_new", v_new, torch.bfloat16),
                            ("k_pool", k_pool, torch.bfloat16), ("v_pool", v_pool, torch.bfloat16),
                            ("seq_lens", seq_lens, torch.int32)):
            if t.dtype != dt or t.device != dev or not t.is_contiguous():
                raise ValueError("%s must be a contiguous %s tensor on %s" % (name, dt, dev))
        if page_table.device != dev:
            raise ValueError("page_table must be on %s" % dev)
        self._bind_table(page_table)
        if k_new.dim() != 3 or tuple(k_new.shape[1:]) != (Hkv, D) or v_new.shape != k_new.shape:
            raise ValueError("k_new and v_new must be [T, %d, %d]" % (Hkv, D))
        if k_pool.dim() != 4 or tuple(k_pool.shape[1:]) != (self.page_size, Hkv, D) \
                or v_pool.shape != k_pool.shape:
            raise ValueError("k_pool and v_pool must be [P, %d, %d, %d]" % (self.page_size, Hkv, D))
        if tuple(seq_lens.shape) != (B,):
            raise ValueError("seq_lens must be [%d]" % B)
        if cu_q_lens is not None:
            if (cu_q_lens.dtype != torch.int32 or tuple(cu_q_lens.shape) != (B + 1,)
                    or cu_q_lens.device != dev or not cu_q_lens.is_contiguous()):
                raise ValueError("cu_q_lens must be a contiguous int32 [%d] tensor" % (B + 1))
        elif k_new.shape[0] != B:
            raise ValueError("without cu_q_lens, k_new must hold one token per request")
        if stream is None:
            stream = torch.cuda.current_stream(dev).cuda_stream
        elif isinstance(stream, torch.cuda.Stream):
            stream = stream.cuda_stream
        _check(self._lib.pa_append_kv(self._h, _ptr(k_new), _ptr(v_new), _ptr(k_pool),
                                      _ptr(v_pool), _ptr(page_table), _ptr(seq_lens),
                                      _ptr(cu_q_lens), ctypes.c_void_p(stream)))

    def profile_start(self, max_runs: int):
        """Record the attention kernel's duration in the next ``max_runs`` runs."""
        _check(self._lib.pa_profile_start(self._h, int(max_runs)))

    def profile_read(self):
        """Returns (summed attention-kernel ms, runs recorded, kernels per run)."""
        ms, n, k = ctypes.c_float(0), ctypes.c_int(0), ctypes.c_int(0)
        _check(self._lib.pa_profile_read(self._h, ctypes.byref(ms), ctypes.byref(n),
                                         ctypes.byref(k)))
        return float(ms.value), int(n.value), int(k.value)

    def status(self, clear: bool = True, stream=None) -> int:
        """Synchronise and read (then clear) the sticky device status word."""
        if stream is None:
            stream = torch.cuda.current_stream().cuda_stream
        v = ctypes.c_uint32(0)
        _check(self._lib.pa_get_status(self._h, ctypes.c_void_p(stream), ctypes.byref(v),
                                       1 if clear else 0))
        return int(v.value)

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pa_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def selftest_wait_timeout(limit_us: int):
    """Run the bounded-wait self-test (pa_selftest_wait_timeout): returns
    (status word, microseconds the short-limit wait took, microseconds the
    production-limit wait took before the abort flag released it)."""
    lib = load_library()
    st = ctypes.c_uint32(0)
    el = (ctypes.c_uint32 * 2)()
    _check(lib.pa_selftest_wait_timeout(int(limit_us), ctypes.byref(st), el))
    return int(st.value), int(el[0]), int(el[1])


def run_noalloc(q, k_pool, v_pool, page_table, seq_lens, cu_q_lens, out, lse, *, heads_kv,
                page_size, capacity, num_pages=0, scale=0.0, stream=None):
    """Call ``pa_run_noalloc``: the attention pass for callers that cannot
    allocate device memory (an engine whose device memory is budgeted by its
    own allocator, a loop that must not stall on an allocation); the
    library's static scratch array replaces the plan's workspace.  Every
    output tensor is passed in; nothing is allocated here or in the library.
    The first call on a device does a one-time set-up there with
    synchronous runtime calls.  Calls that overlap on the GPU race on the
    shared scratch.  Pools are bf16 only.  Read the status word with
    ``noalloc_status`` before the next call, which clears it."""
    lib = load_library()
    B = seq_lens.shape[0]
    Hq, D = q.shape[1], q.shape[2]
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    elif isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    _check(lib.pa_run_noalloc(B, Hq, heads_kv, D, page_size, capacity, int(num_pages),
                              float(scale), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                              _ptr(page_table), _ptr(seq_lens), _ptr(cu_q_lens), _ptr(out),
                              _ptr(lse), ctypes.c_void_p(stream)))


def noalloc_status(clear: bool = True, stream=None) -> int:
    """Synchronise ``stream`` and read (then clear) the status word of the last
    ``pa_run_noalloc`` on the current device (pa_noalloc_get_status)."""
    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    elif isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    v = ctypes.c_uint32(0)
    _check(lib.pa_noalloc_get_status(ctypes.c_void_p(stream), ctypes.byref(v), 1 if clear else 0))
    return int(v.value)
