"""Python handle on the C oracle (``tkv_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product package.

The oracle keeps the whole cache state in numpy arrays owned here, so that a
test can hand it any pre-call state (for instance the state the GPU path held
before a call) and compare the post-call states element by element.

State dictionary (the same keys the GPU export produces):
  n, ft, hw            int32 [S, 4]      live entries / free-stack top / fresh high-water mark
  handle{c}, pos{c}    int32 [S, cap[c]] table of class c (first n entries live)
  score{c}             float32 [S, cap[c]]
  fs{c}                int32 [S, cap[c]] free stack of class c (first ft entries)
  pool{c}              uint8 [S, cap[c], rec_bytes(c)] packed records
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "tkv_oracle.c"
LIB = HERE / "liboracle.so"

ORC_OK, ORC_ERR_INVALID, ORC_ERR_CAPACITY = 0, 1, 2
BITS = (16, 8, 4, 2)


def build(force: bool = False) -> Path:
    """Compile the oracle with IEEE fp32 semantics (no contraction, no fast-math)."""
    if force or not LIB.exists() or LIB.stat().st_mtime < SRC.stat().st_mtime:
        tmp = f"{LIB}.tmp{os.getpid()}"   # per process: concurrent ranks may build at once
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-Wall", "-Wno-unused-function", str(SRC), "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


class _State(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("G", ctypes.c_int32),
        ("D", ctypes.c_int32), ("group", ctypes.c_int32), ("n_protect", ctypes.c_int32),
        ("bits", ctypes.c_int32 * 4), ("cap", ctypes.c_int32 * 4), ("dense", ctypes.c_int32),
        ("pool", ctypes.c_void_p * 4),
        ("n", ctypes.c_void_p), ("ft", ctypes.c_void_p), ("hw", ctypes.c_void_p),
        ("handle", ctypes.c_void_p * 4), ("pos", ctypes.c_void_p * 4),
        ("fs", ctypes.c_void_p * 4), ("score", ctypes.c_void_p * 4),
        ("codec", ctypes.c_int32),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(str(build()))
        L.orc_f32_to_f16_rd.argtypes = [ctypes.c_float]
        L.orc_f32_to_f16_rd.restype = ctypes.c_uint16
        L.orc_f32_to_f16_ru.argtypes = [ctypes.c_float]
        L.orc_f32_to_f16_ru.restype = ctypes.c_uint16
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_record_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.orc_record_bytes.restype = ctypes.c_int
        L.orc_record_bytes_fmt.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.orc_record_bytes_fmt.restype = ctypes.c_int
        L.orc_pack_record_fmt.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3
        L.orc_pack_record_fmt.restype = None
        L.orc_unpack_record_fmt.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3
        L.orc_unpack_record_fmt.restype = None
        L.orc_quantize_group.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_quantize_group.restype = None
        L.orc_pack_record.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3
        L.orc_pack_record.restype = None
        L.orc_unpack_record.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3
        L.orc_unpack_record.restype = None
        L.orc_append.argtypes = [ctypes.POINTER(_State)] + [ctypes.c_void_p] * 4 + [ctypes.c_int]
        L.orc_append.restype = ctypes.c_int
        L.orc_attend.argtypes = [ctypes.POINTER(_State), ctypes.c_void_p, ctypes.c_float,
                                 ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
        L.orc_attend.restype = None
        L.orc_evict.argtypes = [ctypes.POINTER(_State), ctypes.c_int]
        L.orc_evict.restype = ctypes.c_int
        L.orc_evict_window.argtypes = [ctypes.POINTER(_State), ctypes.c_int, ctypes.c_int32]
        L.orc_evict_window.restype = ctypes.c_int
        L.orc_evict_segments.argtypes = [ctypes.POINTER(_State)] + [ctypes.c_void_p] * 4 + [ctypes.c_int]
        L.orc_evict_segments.restype = ctypes.c_int
        L.orc_tbe_schedule.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_void_p]
        L.orc_tbe_schedule.restype = ctypes.c_int
        L.orc_evict_tam.argtypes = [ctypes.POINTER(_State)] + [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_int,
                                                                                      ctypes.c_double]
        L.orc_evict_tam.restype = ctypes.c_int
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_sum_f32_exact.argtypes = [ctypes.c_void_p, ctypes.c_int]
        L.orc_sum_f32_exact.restype = ctypes.c_double
        L.orc_attention_sparsity.argtypes = [ctypes.POINTER(_State), ctypes.c_void_p, ctypes.c_float,
                                             ctypes.c_void_p]
        L.orc_attention_sparsity.restype = None
        L.orc_classify_sparsity.argtypes = [ctypes.c_double] * 3
        L.orc_classify_sparsity.restype = ctypes.c_int
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_round_up.argtypes = [ctypes.c_float]
        L.orc_e4m3_round_up.restype = ctypes.c_uint8
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        for name in ("orc_quantize_group_fp8", "orc_quantize_group_ternary", "orc_quantize_block_nvfp4"):
            getattr(L, name).argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
            getattr(L, name).restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ---------------------------------------------------------------- scalar helpers
def f16_rd(x: float) -> int:
    return lib().orc_f32_to_f16_rd(float(np.float32(x)))


def f16_ru(x: float) -> int:
    return lib().orc_f32_to_f16_ru(float(np.float32(x)))


def f16_value(h: int) -> float:
    return lib().orc_f16_to_f64(h)


def record_bytes(bits: int, D: int = 128, group: int = 32) -> int:
    return lib().orc_record_bytes(bits, D, group)


FMT_FP8, FMT_NVFP4, FMT_TERNARY = 108, 104, 102   # floating-point class record formats


def record_bytes_fmt(fmt: int, D: int = 128, group: int = 32) -> int:
    return lib().orc_record_bytes_fmt(fmt, D, group)


def class_format(bits: int, codec: int) -> int:
    """Record format of a class: bf16 (16), integer codes (8/4/2), or with codec = 1
    the FP codecs (FP8 for 8, NVFP4 for 4, ternary for 2)."""
    return 100 + bits if codec and bits < 16 else bits


def pack_record_fmt(fmt: int, k_bf16: np.ndarray, v_bf16: np.ndarray, D: int = 128, group: int = 32):
    k = np.ascontiguousarray(k_bf16, dtype=np.uint16)
    v = np.ascontiguousarray(v_bf16, dtype=np.uint16)
    rec = np.zeros(record_bytes_fmt(fmt, D, group), dtype=np.uint8)
    lib().orc_pack_record_fmt(fmt, D, group, _ptr(k), _ptr(v), _ptr(rec))
    return rec


def unpack_record_fmt(fmt: int, rec: np.ndarray, D: int = 128, group: int = 32):
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    kh = np.zeros(D, dtype=np.float64)
    vh = np.zeros(D, dtype=np.float64)
    lib().orc_unpack_record_fmt(fmt, D, group, _ptr(rec), _ptr(kh), _ptr(vh))
    return kh, vh


def quantize_group(x, bits: int):
    """x: fp32 values of one group -> (scale_h bits, zero_h bits, codes uint8)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, dtype=np.uint8)
    s = np.zeros(1, dtype=np.uint16)
    z = np.zeros(1, dtype=np.uint16)
    lib().orc_quantize_group(_ptr(x), x.size, bits, _ptr(s), _ptr(z), _ptr(codes))
    return int(s[0]), int(z[0]), codes


def pack_record(bits: int, k_bf16: np.ndarray, v_bf16: np.ndarray, D=128, group=32):
    k = np.ascontiguousarray(k_bf16, dtype=np.uint16)
    v = np.ascontiguousarray(v_bf16, dtype=np.uint16)
    rec = np.zeros(record_bytes(bits, D, group), dtype=np.uint8)
    lib().orc_pack_record(bits, D, group, _ptr(k), _ptr(v), _ptr(rec))
    return rec


def unpack_record(bits: int, rec: np.ndarray, D=128, group=32):
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    kh = np.zeros(D, dtype=np.float64)
    vh = np.zeros(D, dtype=np.float64)
    lib().orc_unpack_record(bits, D, group, _ptr(rec), _ptr(kh), _ptr(vh))
    return kh, vh


def sum_f32_exact(v) -> float:
    """The exact sum of fp32 values (negative and non-finite ones count as 0), rounded
    to the nearest double: the score sums of the TAM budgets."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    return lib().orc_sum_f32_exact(_ptr(a) if a.size else None, int(a.size))


def num_threads() -> int:
    return lib().orc_num_threads()


# ---------------------------------------------------------------- floating-point class codecs
def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    return lib().orc_e4m3_encode(float(np.float32(x)))


def e4m3_round_up(x: float) -> int:
    return lib().orc_e4m3_round_up(float(np.float32(x)))


def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(int(code) & 0xF)


def e2m1_encode(x: float) -> int:
    return lib().orc_e2m1_encode(float(np.float32(x)))


def _quantize_scaled(fn, x, scale_dtype):
    x = np.ascontiguousarray(x, dtype=np.float32)
    sc = np.zeros(1, dtype=scale_dtype)
    codes = np.zeros(len(x), dtype=np.uint8)
    fn(_ptr(x), len(x), _ptr(sc), _ptr(codes))
    return sc[0], codes


def quantize_group_fp8(x):
    """FP8 (E4M3) class group -> (fp16 scale bits, E4M3 codes)."""
    return _quantize_scaled(lib().orc_quantize_group_fp8, x, np.uint16)


def quantize_block_nvfp4(x):
    """NVFP4 block of 16 -> (E4M3 scale code, E2M1 codes)."""
    return _quantize_scaled(lib().orc_quantize_block_nvfp4, x, np.uint8)


def quantize_group_ternary(x):
    """Ternary group -> (fp16 scale bits, codes 0 / 1 (+1) / 3 (-1))."""
    return _quantize_scaled(lib().orc_quantize_group_ternary, x, np.uint16)


def classify_sparsity(s: float, th_r: float, th_t: float) -> int:
    """Thought type (3 T, 1 R, 2 E) of a sparsity value under thresholds th_r <= th_t."""
    return lib().orc_classify_sparsity(float(s), float(th_r), float(th_t))


def tbe_schedule(labels, r0: int = 64, t_keep: int = 16) -> np.ndarray:
    """Retention of each thought segment of one batch row (the last one open) under
    the annealing schedule; -1 keeps the whole segment."""
    lb = np.ascontiguousarray(np.asarray(labels, dtype=np.uint8))
    out = np.zeros(max(len(lb), 1), dtype=np.int32)
    rc = lib().orc_tbe_schedule(_ptr(lb) if len(lb) else 0, len(lb), int(r0), int(t_keep), _ptr(out))
    if rc != 0:
        raise ValueError("invalid schedule arguments")
    return out[:len(lb)]


# ---------------------------------------------------------------- cache model
class OracleCache:
    """Host-side model of one layer's compressed cache."""

    def __init__(self, B, Hkv, G, cap, n_protect, D=128, group=32, bits=BITS, dense=False, codec=0):
        self.B, self.Hkv, self.G, self.D, self.group = B, Hkv, G, D, group
        self.dense = bool(dense)
        self.codec = int(codec)
        self.n_protect = n_protect
        self.bits = tuple(bits)
        self.cap = tuple(int(c) for c in cap)
        self.S = B * Hkv
        S = self.S
        self.state = {"n": np.zeros((S, 4), np.int32), "ft": np.zeros((S, 4), np.int32),
                      "hw": np.zeros((S, 4), np.int32)}
        for c in range(4):
            cc = max(self.cap[c], 1)
            self.state[f"handle{c}"] = np.zeros((S, cc), np.int32)
            self.state[f"pos{c}"] = np.zeros((S, cc), np.int32)
            self.state[f"score{c}"] = np.zeros((S, cc), np.float32)
            self.state[f"fs{c}"] = np.zeros((S, cc), np.int32)
            self.state[f"pool{c}"] = np.zeros(
                (S, cc, record_bytes_fmt(class_format(self.bits[c], self.codec), D, group)), np.uint8)
        self._sync_struct()

    def rec_bytes(self, c):
        return record_bytes_fmt(class_format(self.bits[c], self.codec), self.D, self.group)

    def _sync_struct(self):
        st = _State()
        st.B, st.Hkv, st.G, st.D, st.group = self.B, self.Hkv, self.G, self.D, self.group
        st.n_protect = self.n_protect
        st.dense = int(self.dense)
        st.codec = self.codec
        for c in range(4):
            st.bits[c] = self.bits[c]
            st.cap[c] = self.cap[c]
            st.pool[c] = _ptr(self.state[f"pool{c}"])
            st.handle[c] = _ptr(self.state[f"handle{c}"])
            st.pos[c] = _ptr(self.state[f"pos{c}"])
            st.fs[c] = _ptr(self.state[f"fs{c}"])
            st.score[c] = _ptr(self.state[f"score{c}"])
        st.n = _ptr(self.state["n"])
        st.ft = _ptr(self.state["ft"])
        st.hw = _ptr(self.state["hw"])
        self._st = st

    def load_state(self, state: dict):
        """Replace the whole state by copies of the given arrays (same shapes)."""
        for k, v in state.items():
            if k in self.state:
                self.state[k] = np.ascontiguousarray(np.array(v, dtype=self.state[k].dtype)
                                                     .reshape(self.state[k].shape))
        self._sync_struct()

    def copy_state(self) -> dict:
        return {k: v.copy() for k, v in self.state.items()}

    def append(self, k_bf16: np.ndarray, v_bf16: np.ndarray, cls: np.ndarray, pos: np.ndarray) -> int:
        """k, v: uint16 (bf16 bits) [B, Hkv, T, D]; cls uint8 [B, T]; pos int32 [B, T]."""
        k = np.ascontiguousarray(k_bf16, dtype=np.uint16)
        v = np.ascontiguousarray(v_bf16, dtype=np.uint16)
        cls = np.ascontiguousarray(cls, dtype=np.uint8)
        pos = np.ascontiguousarray(pos, dtype=np.int32)
        T = k.shape[2]
        assert k.shape == (self.B, self.Hkv, T, self.D) and cls.shape == (self.B, T)
        return lib().orc_append(ctypes.byref(self._st), _ptr(k), _ptr(v), _ptr(cls), _ptr(pos), T)

    def attend(self, q_bf16: np.ndarray, softmax_scale: float, s_dbg: int = -1):
        """q: uint16 (bf16 bits) [B, Hkv*G, D] -> out fp32 [B, Hkv*G, D] (and p of s_dbg)."""
        q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
        assert q.shape == (self.B, self.Hkv * self.G, self.D)
        out = np.zeros(q.shape, dtype=np.float32)
        p = None
        pp = None
        if s_dbg >= 0:
            N = int(self.state["n"][s_dbg].sum())
            p = np.zeros((self.G, max(N, 1)), dtype=np.float64)
            pp = _ptr(p)
        lib().orc_attend(ctypes.byref(self._st), _ptr(q), float(softmax_scale), _ptr(out),
                         int(s_dbg), pp)
        return (out, p) if s_dbg >= 0 else out

    def attention_sparsity(self, q_bf16: np.ndarray, softmax_scale: float) -> np.ndarray:
        """1 - H(p) / ln N per stream and query head for the step's query -> [S, G]."""
        q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
        assert q.shape == (self.B, self.Hkv * self.G, self.D)
        out = np.zeros((self.S, self.G), dtype=np.float64)
        lib().orc_attention_sparsity(ctypes.byref(self._st), _ptr(q), float(softmax_scale), _ptr(out))
        return out

    def evict(self, budget: int) -> int:
        return lib().orc_evict(ctypes.byref(self._st), int(budget))

    def evict_window(self, budget: int, keep_from: int) -> int:
        """Top-k eviction whose candidates are the positions in [n_protect, keep_from):
        the local window (positions >= keep_from) is kept as well."""
        return lib().orc_evict_window(ctypes.byref(self._st), int(budget), int(keep_from))

    def evict_segments(self, seg_start: np.ndarray, seg_label: np.ndarray, seg_keep: np.ndarray,
                       nseg: np.ndarray) -> int:
        """Segment-level eviction.  seg_start int32 / seg_label uint8 / seg_keep int32
        [B, max_seg] (row b: the thought segments of batch row b), nseg int32 [B]."""
        st_ = np.ascontiguousarray(seg_start, dtype=np.int32)
        lb = np.ascontiguousarray(seg_label, dtype=np.uint8)
        kp = np.ascontiguousarray(seg_keep, dtype=np.int32)
        ns = np.ascontiguousarray(nseg, dtype=np.int32)
        assert st_.ndim == 2 and st_.shape[0] == self.B and lb.shape == st_.shape == kp.shape
        assert ns.shape == (self.B,)
        return lib().orc_evict_segments(ctypes.byref(self._st), _ptr(st_), _ptr(lb), _ptr(kp), _ptr(ns),
                                        st_.shape[1])

    def evict_tam(self, seg_start: np.ndarray, seg_label: np.ndarray, nseg: np.ndarray, budget: int,
                  c: float) -> int:
        """Thought-aware budgets (t_j proportional to sqrt(w_j) n_j) with pivotal tokens
        (score >= c * mean) kept; segment arrays as for evict_segments."""
        st_ = np.ascontiguousarray(seg_start, dtype=np.int32)
        lb = np.ascontiguousarray(seg_label, dtype=np.uint8)
        ns = np.ascontiguousarray(nseg, dtype=np.int32)
        assert st_.ndim == 2 and st_.shape[0] == self.B and lb.shape == st_.shape and ns.shape == (self.B,)
        return lib().orc_evict_tam(ctypes.byref(self._st), _ptr(st_), _ptr(lb), _ptr(ns), st_.shape[1],
                                   int(budget), float(c))

    # -- convenience views
    def live(self, s: int, c: int):
        n = self.state["n"][s, c]
        return (self.state[f"handle{c}"][s, :n], self.state[f"pos{c}"][s, :n],
                self.state[f"score{c}"][s, :n])
