"""Thin ctypes binding of libtkv (include/tkv.h).

Argument marshalling only: torch tensors provide device memory and the current
CUDA stream; every step of the decode path runs in the library's kernels.
There is no fallback: if libtkv.so is missing or no CUDA device is present,
the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

import numpy as np
import torch

# TKV_LIBRARY selects another build of the library (e.g. libtkv_debug.so, the
# bounds-checking build) for the whole process; by default the release build.
LIB_PATH = Path(os.environ.get("TKV_LIBRARY") or (Path(__file__).resolve().parent / "libtkv.so"))

TKV_OK, TKV_ERR_INVALID, TKV_ERR_CAPACITY, TKV_ERR_CUDA, TKV_ERR_TIMEOUT = range(5)
STATUS_NAMES = {0: "TKV_OK", 1: "TKV_ERR_INVALID", 2: "TKV_ERR_CAPACITY", 3: "TKV_ERR_CUDA",
                4: "TKV_ERR_TIMEOUT"}
BITS = (16, 8, 4, 2)


class TkvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class TkvConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("G", ctypes.c_int32),
                ("D", ctypes.c_int32), ("group", ctypes.c_int32), ("bits", ctypes.c_int32 * 4),
                ("n_protect", ctypes.c_int32), ("cap", ctypes.c_int32 * 4),
                ("max_append", ctypes.c_int32), ("dense", ctypes.c_int32),
                ("attn_kernel", ctypes.c_int32), ("codec", ctypes.c_int32)]


class TkvLayout(ctypes.Structure):
    _fields_ = [("n", ctypes.c_size_t), ("ft", ctypes.c_size_t), ("hw", ctypes.c_size_t),
                ("err", ctypes.c_size_t), ("handle", ctypes.c_size_t * 4),
                ("pos", ctypes.c_size_t * 4), ("score", ctypes.c_size_t * 4),
                ("fs", ctypes.c_size_t * 4), ("pool", ctypes.c_size_t * 4),
                ("rec_bytes", ctypes.c_int32 * 4), ("state_bytes", ctypes.c_size_t),
                ("total_bytes", ctypes.c_size_t)]


EXPORTS = ["tkv_workspace_bytes", "tkv_create", "tkv_destroy", "tkv_reset", "tkv_get_layout",
           "tkv_quantize_append", "tkv_quantize_append_noalloc", "tkv_decode_attention", "tkv_evict_compact", "tkv_poll_error",
           "tkv_export_state", "tkv_import_state", "tkv_launch_count", "tkv_last_error_string",
           "tkv_selftest_wait_timeout", "tkv_evict_segments", "tkv_tbe_schedule",
           "tkv_evict_tam", "tkv_evict_compact_window", "tkv_decode_attention_sparsity", "tkv_decode_step"]

_lib = None


def lib() -> ctypes.CDLL:
    """Load libtkv.so (built by reasoning_model_kv_b200.build); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m reasoning_model_kv_b200.build`")
    L = ctypes.CDLL(str(LIB_PATH))
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    P = ctypes.POINTER
    L.tkv_workspace_bytes.argtypes = [P(TkvConfig)]
    L.tkv_workspace_bytes.restype = sz
    L.tkv_create.argtypes = [P(TkvConfig), vp, sz, P(vp)]
    L.tkv_destroy.argtypes = [vp]
    L.tkv_reset.argtypes = [vp, vp]
    L.tkv_get_layout.argtypes = [vp, P(TkvLayout)]
    L.tkv_quantize_append.argtypes = [vp, vp, vp, vp, vp, i32, vp]
    L.tkv_quantize_append_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, vp]
    L.tkv_decode_attention.argtypes = [vp, vp, ctypes.c_float, vp, vp]
    L.tkv_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp]
    L.tkv_decode_attention_sparsity.argtypes = [vp, vp, ctypes.c_float, vp, vp, vp, ctypes.c_float,
                                                ctypes.c_float, vp]
    L.tkv_decode_attention_sparsity.restype = ctypes.c_int
    L.tkv_evict_compact.argtypes = [vp, i32, vp]
    L.tkv_poll_error.argtypes = [vp, vp]
    L.tkv_export_state.argtypes = [vp, vp, vp]
    L.tkv_import_state.argtypes = [vp, vp, vp]
    L.tkv_launch_count.argtypes = [vp]
    L.tkv_selftest_wait_timeout.argtypes = [vp, ctypes.c_int64, vp]
    L.tkv_selftest_wait_timeout.restype = ctypes.c_int
    L.tkv_evict_segments.argtypes = [vp, vp, vp, vp, vp, i32, vp]
    L.tkv_evict_segments.restype = ctypes.c_int
    L.tkv_tbe_schedule.argtypes = [vp, i32, i32, i32, vp]
    L.tkv_tbe_schedule.restype = ctypes.c_int
    L.tkv_evict_tam.argtypes = [vp, vp, vp, vp, i32, i32, ctypes.c_double, vp]
    L.tkv_evict_tam.restype = ctypes.c_int
    L.tkv_evict_compact_window.argtypes = [vp, i32, i32, vp]
    L.tkv_evict_compact_window.restype = ctypes.c_int
    L.tkv_launch_count.restype = ctypes.c_int64
    L.tkv_last_error_string.restype = ctypes.c_char_p
    for name in ("tkv_create", "tkv_destroy", "tkv_reset", "tkv_get_layout", "tkv_quantize_append",
                 "tkv_quantize_append_noalloc",
                 "tkv_decode_attention", "tkv_decode_step", "tkv_evict_compact", "tkv_poll_error", "tkv_export_state",
                 "tkv_import_state"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int):
    if status != TKV_OK:
        raise TkvError(status, lib().tkv_last_error_string().decode())


def make_config(B, Hkv, G, cap, n_protect, max_append=1, D=128, group=32, dense=False,
                attn_kernel=0, codec=0) -> TkvConfig:
    cfg = TkvConfig()
    cfg.B, cfg.Hkv, cfg.G, cfg.D, cfg.group = B, Hkv, G, D, group
    for i in range(4):
        cfg.bits[i] = BITS[i]
        cfg.cap[i] = int(cap[i])
    cfg.n_protect = n_protect
    cfg.max_append = max_append
    cfg.dense = int(bool(dense))
    cfg.attn_kernel = int(attn_kernel)
    cfg.codec = int(codec)
    return cfg


def tkv_workspace_bytes(cfg: TkvConfig) -> int:
    return lib().tkv_workspace_bytes(ctypes.byref(cfg))


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dptr(t: torch.Tensor, dtype, name: str) -> int:
    if not t.is_cuda:
        raise TkvError(TKV_ERR_INVALID, f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TkvError(TKV_ERR_INVALID, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise TkvError(TKV_ERR_INVALID, f"{name} must be contiguous")
    return t.data_ptr()


class TkvCache:
    """One layer's compressed KV cache: a device workspace owned by torch plus the
    library's cache object.  Methods mirror the C ABI names."""

    def __init__(self, B, Hkv, G, cap, n_protect, max_append=1, device="cuda", dense=False, attn_kernel=0,
                 codec=0):
        self.cfg = make_config(B, Hkv, G, cap, n_protect, max_append, dense=dense, attn_kernel=attn_kernel,
                               codec=codec)
        self.dense = bool(dense)
        self.attn_kernel = int(attn_kernel)
        self.codec = int(codec)
        self.B, self.Hkv, self.G, self.S = B, Hkv, G, B * Hkv
        self.cap = tuple(int(c) for c in cap)
        self.n_protect, self.max_append = n_protect, max_append
        nbytes = tkv_workspace_bytes(self.cfg)
        if nbytes == 0:
            raise TkvError(TKV_ERR_INVALID, lib().tkv_last_error_string().decode())
        self.workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.workspace.data_ptr()
        self._pad = (-base) % 256
        h = ctypes.c_void_p()
        _check(lib().tkv_create(ctypes.byref(self.cfg), base + self._pad, nbytes, ctypes.byref(h)))
        self._h = h
        self.layout = TkvLayout()
        _check(lib().tkv_get_layout(self._h, ctypes.byref(self.layout)))
        self.reset()

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.tkv_destroy(h)
            self._h = None

    # -- the three calls of the decode path
    def quantize_append(self, k: torch.Tensor, v: torch.Tensor, cls: torch.Tensor,
                        pos: torch.Tensor, stream=None):
        T = k.shape[2]
        if k.shape != (self.B, self.Hkv, T, 128) or v.shape != k.shape:
            raise TkvError(TKV_ERR_INVALID, f"k/v must be [B, Hkv, T, 128], got {tuple(k.shape)}")
        if cls.shape != (self.B, T) or pos.shape != (self.B, T):
            raise TkvError(TKV_ERR_INVALID, "cls/pos must be [B, T]")
        _check(lib().tkv_quantize_append(self._h, _dptr(k, torch.bfloat16, "k"),
                                         _dptr(v, torch.bfloat16, "v"),
                                         _dptr(cls, torch.uint8, "cls"),
                                         _dptr(pos, torch.int32, "pos"), T, _stream(stream)))

    def quantize_append_noalloc(self, k: torch.Tensor, v: torch.Tensor, cls: torch.Tensor,
                                pos: torch.Tensor, stream=None):
        """Same as quantize_append, using the library's fixed device scratch instead of
        the workspace's (for callers that cannot allocate; B*(T+4) <= 524288)."""
        T = k.shape[2]
        if k.shape != (self.B, self.Hkv, T, 128) or v.shape != k.shape:
            raise TkvError(TKV_ERR_INVALID, f"k/v must be [B, Hkv, T, 128], got {tuple(k.shape)}")
        if cls.shape != (self.B, T) or pos.shape != (self.B, T):
            raise TkvError(TKV_ERR_INVALID, "cls/pos must be [B, T]")
        _check(lib().tkv_quantize_append_noalloc(self._h, _dptr(k, torch.bfloat16, "k"),
                                                 _dptr(v, torch.bfloat16, "v"),
                                                 _dptr(cls, torch.uint8, "cls"),
                                                 _dptr(pos, torch.int32, "pos"), T, _stream(stream)))

    def decode_attention(self, q: torch.Tensor, softmax_scale: float, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
        if q.shape != (self.B, self.Hkv * self.G, 128):
            raise TkvError(TKV_ERR_INVALID, f"q must be [B, Hkv*G, 128], got {tuple(q.shape)}")
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        _check(lib().tkv_decode_attention(self._h, _dptr(q, torch.bfloat16, "q"),
                                          float(softmax_scale), _dptr(out, torch.float32, "out"),
                                          _stream(stream)))
        return out

    def decode_step(self, k: torch.Tensor, v: torch.Tensor, cls: torch.Tensor, pos: torch.Tensor,
                    q: torch.Tensor, softmax_scale: float, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
        """One decode step with its new token: quantize_append of k, v [B, Hkv, 128] (cls,
        pos [B]) followed by decode_attention of q, in one call."""
        if k.shape != (self.B, self.Hkv, 128) or v.shape != k.shape:
            raise TkvError(TKV_ERR_INVALID, f"k/v must be [B, Hkv, 128], got {tuple(k.shape)}")
        if cls.shape != (self.B,) or pos.shape != (self.B,):
            raise TkvError(TKV_ERR_INVALID, "cls/pos must be [B]")
        if q.shape != (self.B, self.Hkv * self.G, 128):
            raise TkvError(TKV_ERR_INVALID, f"q must be [B, Hkv*G, 128], got {tuple(q.shape)}")
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        _check(lib().tkv_decode_step(self._h, _dptr(k, torch.bfloat16, "k"), _dptr(v, torch.bfloat16, "v"),
                                     _dptr(cls, torch.uint8, "cls"), _dptr(pos, torch.int32, "pos"),
                                     _dptr(q, torch.bfloat16, "q"), float(softmax_scale),
                                     _dptr(out, torch.float32, "out"), _stream(stream)))
        return out

    def decode_attention_sparsity(self, q: torch.Tensor, softmax_scale: float, th_r: float = 0.5,
                                  th_t: float = 0.7, out: torch.Tensor | None = None, stream=None):
        """decode_attention plus the per-(stream, head) attention sparsity 1 - H(p)/ln N
        and its thought class (3 T if >= th_t, 1 R if >= th_r, else 2 E); returns
        (out, sparsity [B, Hkv*G] fp32, thought class [B, Hkv*G] uint8)."""
        if q.shape != (self.B, self.Hkv * self.G, 128):
            raise TkvError(TKV_ERR_INVALID, f"q must be [B, Hkv*G, 128], got {tuple(q.shape)}")
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        sp = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
        cls = torch.empty(q.shape[:2], dtype=torch.uint8, device=q.device)
        _check(lib().tkv_decode_attention_sparsity(self._h, _dptr(q, torch.bfloat16, "q"), float(softmax_scale),
                                                   _dptr(out, torch.float32, "out"),
                                                   _dptr(sp, torch.float32, "sparsity"),
                                                   _dptr(cls, torch.uint8, "thought"), float(th_r), float(th_t),
                                                   _stream(stream)))
        return out, sp, cls

    def evict_compact(self, budget: int, stream=None):
        _check(lib().tkv_evict_compact(self._h, int(budget), _stream(stream)))

    def evict_compact_window(self, budget: int, keep_from: int, stream=None):
        """Top-k eviction that also keeps every entry at a position >= keep_from
        (the local window of recent tokens)."""
        _check(lib().tkv_evict_compact_window(self._h, int(budget), int(keep_from), _stream(stream)))

    def evict_segments(self, seg_start: torch.Tensor, seg_label: torch.Tensor, seg_keep: torch.Tensor,
                       nseg: torch.Tensor, stream=None):
        """Segment-level eviction: seg_start int32 / seg_label uint8 / seg_keep int32
        [B, max_seg] and nseg int32 [B], all on the device."""
        if seg_start.dim() != 2 or seg_start.shape[0] != self.B:
            raise TkvError(TKV_ERR_INVALID, "seg_start must be [B, max_seg]")
        shape = tuple(seg_start.shape)
        for t, name in ((seg_label, "seg_label"), (seg_keep, "seg_keep")):
            if tuple(t.shape) != shape:
                raise TkvError(TKV_ERR_INVALID, f"{name} must be [B, max_seg]")
        if tuple(nseg.shape) != (self.B,):
            raise TkvError(TKV_ERR_INVALID, "nseg must be [B]")
        _check(lib().tkv_evict_segments(self._h, _dptr(seg_start, torch.int32, "seg_start"),
                                        _dptr(seg_label, torch.uint8, "seg_label"),
                                        _dptr(seg_keep, torch.int32, "seg_keep"),
                                        _dptr(nseg, torch.int32, "nseg"), shape[1], _stream(stream)))

    def evict_tam(self, seg_start: torch.Tensor, seg_label: torch.Tensor, nseg: torch.Tensor, budget: int,
                  c: float, stream=None):
        """Thought-aware segment budgets with pivotal tokens (score >= c * mean) kept;
        seg_start int32 / seg_label uint8 [B, max_seg], nseg int32 [B], on the device."""
        if seg_start.dim() != 2 or seg_start.shape[0] != self.B or tuple(seg_label.shape) != tuple(seg_start.shape):
            raise TkvError(TKV_ERR_INVALID, "seg_start and seg_label must be [B, max_seg]")
        if tuple(nseg.shape) != (self.B,):
            raise TkvError(TKV_ERR_INVALID, "nseg must be [B]")
        _check(lib().tkv_evict_tam(self._h, _dptr(seg_start, torch.int32, "seg_start"),
                                   _dptr(seg_label, torch.uint8, "seg_label"), _dptr(nseg, torch.int32, "nseg"),
                                   seg_start.shape[1], int(budget), float(c), _stream(stream)))

    # -- housekeeping
    def reset(self, stream=None):
        _check(lib().tkv_reset(self._h, _stream(stream)))

    def poll_error(self, stream=None) -> int:
        """Synchronise and return (and clear) the first device-side status."""
        st = lib().tkv_poll_error(self._h, _stream(stream))
        if st == TKV_ERR_CUDA:
            _check(st)
        return st

    def selftest_wait_timeout(self, limit_cycles: int, stream=None):
        """Run the bounded-wait self-test (a wait that must give up); the next
        poll_error() returns TKV_ERR_TIMEOUT."""
        _check(lib().tkv_selftest_wait_timeout(self._h, int(limit_cycles), _stream(stream)))

    def launch_count(self) -> int:
        return lib().tkv_launch_count(self._h)

    def state_views(self) -> dict:
        """Zero-copy torch views of the state arrays inside the workspace."""
        L = self.layout
        ws = self.workspace[self._pad:]
        S = self.S

        def view(off, count, dtype, shape):
            nbytes = count * torch.empty((), dtype=dtype).element_size()
            return ws[off:off + nbytes].view(dtype).view(*shape)

        out = {"n": view(L.n, S * 4, torch.int32, (S, 4)),
               "ft": view(L.ft, S * 4, torch.int32, (S, 4)),
               "hw": view(L.hw, S * 4, torch.int32, (S, 4))}
        for c in range(4):
            cc = self.cap[c]
            out[f"handle{c}"] = view(L.handle[c], S * cc, torch.int32, (S, cc))
            out[f"pos{c}"] = view(L.pos[c], S * cc, torch.int32, (S, cc))
            out[f"score{c}"] = view(L.score[c], S * cc, torch.float32, (S, cc))
            out[f"fs{c}"] = view(L.fs[c], S * cc, torch.int32, (S, cc))
            rb = L.rec_bytes[c]
            out[f"pool{c}"] = ws[L.pool[c]:L.pool[c] + S * cc * rb].view(S, cc, rb)
        return out

    def _state_arrays(self, buf: np.ndarray) -> dict:
        """Numpy views of the state arrays inside a host copy of the state region
        (the tkv_layout offsets; same keys and shapes as state_views)."""
        L = self.layout
        S = self.S

        def view(off, count, dtype, shape):
            nbytes = count * np.dtype(dtype).itemsize
            return buf[off:off + nbytes].view(dtype).reshape(shape)

        out = {"n": view(L.n, S * 4, np.int32, (S, 4)),
               "ft": view(L.ft, S * 4, np.int32, (S, 4)),
               "hw": view(L.hw, S * 4, np.int32, (S, 4))}
        for c in range(4):
            cc = self.cap[c]
            out[f"handle{c}"] = view(L.handle[c], S * cc, np.int32, (S, cc))
            out[f"pos{c}"] = view(L.pos[c], S * cc, np.int32, (S, cc))
            out[f"score{c}"] = view(L.score[c], S * cc, np.float32, (S, cc))
            out[f"fs{c}"] = view(L.fs[c], S * cc, np.int32, (S, cc))
            rb = L.rec_bytes[c]
            out[f"pool{c}"] = view(L.pool[c], S * cc * rb, np.uint8, (S, cc, rb))
        return out

    def export_state(self, streams=None) -> dict:
        """Host (numpy) copy of the state.  The whole state goes through the C ABI's
        tkv_export_state (one copy of the state region); a subset of streams is read
        through device views of the workspace instead, which avoids copying every
        stream of a large cache to the host."""
        if streams is None:
            buf = np.empty(self.layout.state_bytes, dtype=np.uint8)
            _check(lib().tkv_export_state(self._h, buf.ctypes.data, _stream()))
            return self._state_arrays(buf)
        torch.cuda.current_stream().synchronize()
        v = self.state_views()
        idx = torch.as_tensor(list(streams), device=self.workspace.device)
        return {k: t.index_select(0, idx).cpu().numpy() for k, t in v.items()}

    def import_state(self, state: dict):
        """Load state arrays (all streams; keys as export_state returns them) through
        the C ABI's tkv_import_state.  Keys that are absent keep their current
        contents."""
        buf = np.empty(self.layout.state_bytes, dtype=np.uint8)
        _check(lib().tkv_export_state(self._h, buf.ctypes.data, _stream()))
        arrs = self._state_arrays(buf)
        for k, arr in state.items():
            if k not in arrs:
                raise TkvError(TKV_ERR_INVALID, f"unknown state array {k}")
            a = np.asarray(arr)
            if a.shape != arrs[k].shape:
                raise TkvError(TKV_ERR_INVALID, f"{k} must have shape {arrs[k].shape}, got {a.shape}")
            arrs[k][...] = a.view(arrs[k].dtype) if a.dtype.itemsize == arrs[k].dtype.itemsize else a
        _check(lib().tkv_import_state(self._h, buf.ctypes.data, _stream()))


# Module-level aliases with the C ABI's names.
def tkv_quantize_append(cache: TkvCache, k, v, cls, pos, stream=None):
    return cache.quantize_append(k, v, cls, pos, stream)


def tkv_decode_attention(cache: TkvCache, q, softmax_scale, out=None, stream=None):
    return cache.decode_attention(q, softmax_scale, out, stream)


def tkv_decode_step(cache: TkvCache, k, v, cls, pos, q, softmax_scale, out=None, stream=None):
    return cache.decode_step(k, v, cls, pos, q, softmax_scale, out, stream)


def tkv_evict_compact(cache: TkvCache, budget, stream=None):
    return cache.evict_compact(budget, stream)


def tkv_evict_compact_window(cache: TkvCache, budget, keep_from, stream=None):
    return cache.evict_compact_window(budget, keep_from, stream)


def tkv_evict_segments(cache: TkvCache, seg_start, seg_label, seg_keep, nseg, stream=None):
    return cache.evict_segments(seg_start, seg_label, seg_keep, nseg, stream)


def tkv_evict_tam(cache: TkvCache, seg_start, seg_label, nseg, budget, c, stream=None):
    return cache.evict_tam(seg_start, seg_label, nseg, budget, c, stream)


def tkv_tbe_schedule(labels, r0: int = 64, t_keep: int = 16):
    """Retention of each thought segment of one batch row (host computation in the
    library): a list of ints, -1 keeps the segment whole."""
    lab = (ctypes.c_uint8 * max(len(labels), 1))(*[int(x) for x in labels])
    out = (ctypes.c_int32 * max(len(labels), 1))()
    _check(lib().tkv_tbe_schedule(ctypes.addressof(lab), len(labels), int(r0), int(t_keep),
                                  ctypes.addressof(out)))
    return [int(out[i]) for i in range(len(labels))]
