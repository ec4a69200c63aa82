"""Python binding of libnq (include/nq.h): argument marshalling only.

Every step of the path runs in the CUDA library; this module turns torch
tensors into pointers, strides and the current CUDA stream, and raises when a
call returns a non-OK status.  There is no fallback: if libnq.so is missing
or the device is not CUDA, the calls fail loudly.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(HERE, "libnq.so")
D = 128

NQ_OK, NQ_ERR_INVALID, NQ_ERR_WORKSPACE, NQ_ERR_CUDA, NQ_ERR_UNSUPPORTED = range(5)


class NQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libnq status {status}: {msg}")
        self.status = status


class KVStrides(ctypes.Structure):
    _fields_ = [("unit", ctypes.c_int64), ("head", ctypes.c_int64), ("token", ctypes.c_int64)]


class Packed(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p),
                ("unit_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64),
                ("bits", ctypes.c_int32)]


class PackedExact(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("sigma", ctypes.c_void_p),
                ("unit_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64),
                ("bits", ctypes.c_int32)]


_lib = None

EXPORTS = (
    "nq_last_error", "nq_version", "nq_packed_bytes_per_vector", "nq_rope_tables_bytes",
    "nq_rope_tables_fill_host", "nq_score_workspace_bytes", "nq_score", "nq_score_static",
    "nq_kept_count",
    "nq_select", "nq_encode", "nq_decode", "nq_e8_quantise", "nq_attend_workspace_bytes",
    "nq_attend", "nq_device_error", "nq_entropy_streams", "nq_entropy_max_words",
    "nq_entropy_workspace_bytes", "nq_entropy_encode", "nq_entropy_decode",
    "nq_packed_exact_bytes_per_vector", "nq_encode_exact", "nq_decode_exact",
    "nq_e8_box_quantise", "nq_set_decode_engine", "nq_get_decode_engine",
)


def lib() -> ctypes.CDLL:
    """Load libnq.so from the package directory (built by build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(SO_PATH):
        raise ImportError(f"libnq.so not built at {SO_PATH}; run python -m e8_lattice_vector_nq_b200.build")
    L = ctypes.CDLL(SO_PATH)
    P, i64, i32, sz, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_double
    PK = ctypes.POINTER(Packed)
    PX = ctypes.POINTER(PackedExact)
    sig = {
        "nq_last_error": (ctypes.c_char_p, []),
        "nq_version": (i32, []),
        "nq_packed_bytes_per_vector": (i64, [i32]),
        "nq_rope_tables_bytes": (sz, [i64]),
        "nq_rope_tables_fill_host": (i32, [dbl, i64, P, sz]),
        "nq_score_workspace_bytes": (sz, [i32, i32]),
        "nq_score": (i32, [P, KVStrides, i32, i32, i64, i32, P, P, sz, P]),
        "nq_score_static": (i32, [P, KVStrides, i32, i32, i64, i32, P, P]),
        "nq_kept_count": (i64, [i64, i64, i32]),
        "nq_select": (i32, [P, i32, i64, i32, i32, P, i64, P]),
        "nq_encode": (i32, [P, KVStrides, P, KVStrides, i32, i32, i64, i64, P, i64, i64, P, i64,
                            PK, PK, i64, P]),
        "nq_decode": (i32, [PK, PK, i32, i32, i64, i64, P, i64, i64, P, i64, P, KVStrides, P,
                            KVStrides, P]),
        "nq_e8_quantise": (i32, [P, i64, i32, P, P, P]),
        "nq_attend_workspace_bytes": (sz, [i32, i32, i32, i64]),
        "nq_attend": (i32, [P, i32, i32, i32, PK, PK, i64, i64, P, i64, i64, P, i64,
                            ctypes.c_float, P, P, P, sz, P]),
        "nq_device_error": (i32, [ctypes.POINTER(ctypes.c_uint32)]),
        "nq_set_decode_engine": (i32, [i32]),
        "nq_get_decode_engine": (i32, []),
        "nq_entropy_streams": (i64, [i32, i32, i64]),
        "nq_entropy_max_words": (i64, [i32, i32, i64]),
        "nq_entropy_workspace_bytes": (sz, [i32, i32, i64]),
        "nq_entropy_encode": (i32, [PK, i32, i32, i64, i64, i32, P, P, P, i64, P, sz, P]),
        "nq_entropy_decode": (i32, [P, P, P, i32, i32, i64, i32, PK, i64, P]),
        "nq_packed_exact_bytes_per_vector": (i64, [i32]),
        "nq_encode_exact": (i32, [P, KVStrides, P, KVStrides, i32, i32, i64, i64, P, i64, i64, P,
                                  i64, PX, PX, i64, P]),
        "nq_decode_exact": (i32, [PX, PX, i32, i32, i64, i64, P, i64, i64, P, i64, P, KVStrides,
                                  P, KVStrides, P]),
        "nq_e8_box_quantise": (i32, [P, i64, i32, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int):
    if status != NQ_OK:
        raise NQError(status, lib().nq_last_error().decode())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libnq works on CUDA tensors only (no CPU path)")


def _require_device_readable(*ts):
    """CUDA tensors, or pinned host tensors: with unified addressing the
    kernels read pinned host memory in place over the bus (no CPU arithmetic)."""
    for t in ts:
        if t is not None and not (t.is_cuda or t.is_pinned()):
            raise ValueError("libnq reads CUDA tensors or pinned host tensors only (no CPU path)")


def kv_strides(t: torch.Tensor) -> KVStrides:
    """Strides of a [units][heads][tokens][128] bf16 tensor (last dim contiguous)."""
    if t.dim() != 4 or t.shape[-1] != D or t.stride(-1) != 1 or t.dtype != torch.bfloat16:
        raise ValueError("expected bf16 [units, heads, tokens, 128] with a contiguous last dim")
    return KVStrides(t.stride(0), t.stride(1), t.stride(2))


# ------------------------------------------------------------ packed store
@dataclass
class PackedStore:
    """Device arrays of one packed K or V store: codes [units][heads][cap][4*bits]
    (uint32 words held in an int32 tensor) and meta [units][heads][cap]."""

    codes: torch.Tensor
    meta: torch.Tensor
    bits: int

    @classmethod
    def empty(cls, units: int, heads: int, cap: int, bits: int, device="cuda") -> "PackedStore":
        codes = torch.empty(units, heads, cap, 4 * bits, dtype=torch.int32, device=device)
        meta = torch.empty(units, heads, cap, dtype=torch.int32, device=device)
        return cls(codes, meta, bits)

    def select_units(self, sl) -> "PackedStore":
        return PackedStore(self.codes[sl], self.meta[sl], self.bits)

    def desc(self) -> Packed:
        assert self.codes.stride(1) == self.meta.stride(1) * 4 * self.bits
        assert self.codes.stride(0) == self.meta.stride(0) * 4 * self.bits
        return Packed(self.codes.data_ptr(), self.meta.data_ptr(), self.meta.stride(0),
                      self.meta.stride(1), self.bits)

    @property
    def nbytes(self) -> int:
        return self.codes.numel() * 4 + self.meta.numel() * 4


@dataclass
class ExactStore:
    """Device arrays of one exact-layout store (nq.h, nq_packed_exact): codes
    [units][heads][cap][4*bits] (uint32 words in an int32 tensor; the low bit
    of code 8g+7 holds group g's coset bit) and sigma [units][heads][cap]
    (fp16 scale bits in an int16 tensor)."""

    codes: torch.Tensor
    sigma: torch.Tensor
    bits: int

    @classmethod
    def empty(cls, units: int, heads: int, cap: int, bits: int, device="cuda") -> "ExactStore":
        codes = torch.empty(units, heads, cap, 4 * bits, dtype=torch.int32, device=device)
        sigma = torch.empty(units, heads, cap, dtype=torch.int16, device=device)
        return cls(codes, sigma, bits)

    def select_units(self, sl) -> "ExactStore":
        return ExactStore(self.codes[sl], self.sigma[sl], self.bits)

    def desc(self) -> PackedExact:
        assert self.codes.stride(1) == self.sigma.stride(1) * 4 * self.bits
        assert self.codes.stride(0) == self.sigma.stride(0) * 4 * self.bits
        return PackedExact(self.codes.data_ptr(), self.sigma.data_ptr(), self.sigma.stride(0),
                           self.sigma.stride(1), self.bits)

    def codes_store(self) -> PackedStore:
        """The codes as an nq_packed for the entropy stage (which reads codes
        only; the meta array given is a placeholder that is never read)."""
        meta = torch.empty(self.sigma.shape, dtype=torch.int32, device=self.codes.device)
        return PackedStore(self.codes, meta, self.bits)

    @property
    def nbytes(self) -> int:
        return self.codes.numel() * 4 + self.sigma.numel() * 2


# -------------------------------------------------------------- RoPE tables
def rope_tables(theta: float, max_pos: int, device="cuda") -> torch.Tensor:
    """Two-level fp32 cos/sin tables built on the host by the library, copied to the device."""
    L = lib()
    nbytes = L.nq_rope_tables_bytes(int(max_pos))
    host = torch.empty(nbytes // 4, dtype=torch.float32)
    _check(L.nq_rope_tables_fill_host(float(theta), int(max_pos), _ptr(host), nbytes))
    return host.to(device)


# --------------------------------------------------------------- the calls
def kept_count(T: int, W: int, evict_pct: int) -> int:
    return int(lib().nq_kept_count(int(T), int(W), int(evict_pct)))


def score_workspace(units: int, heads: int, device="cuda") -> torch.Tensor:
    n = lib().nq_score_workspace_bytes(int(units), int(heads))
    return torch.empty(max(n, 16) // 4, dtype=torch.float32, device=device)


def nq_score(K: torch.Tensor, W: int, scores: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """scores[u][t] (fp64) of K [units][heads][T][128] (see nq.h, nq_score)."""
    _require_cuda(K)
    units, heads, T, _ = K.shape
    if scores is None:
        scores = torch.empty(units, T, dtype=torch.float64, device=K.device)
    if ws is None:
        ws = score_workspace(units, heads, K.device)
    assert scores.is_contiguous() and scores.dtype == torch.float64
    _check(lib().nq_score(_ptr(K), kv_strides(K), units, heads, T, int(W), _ptr(scores), _ptr(ws),
                          ws.numel() * ws.element_size(), _stream(stream)))
    return scores


def nq_score_static(K: torch.Tensor, W: int, scores: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Same scores as nq_score without a caller workspace: for callers that
    cannot allocate device memory (see nq.h, nq_score_static).  Calls that
    overlap on one GPU race on the library's shared scratch."""
    _require_cuda(K)
    units, heads, T, _ = K.shape
    if scores is None:
        scores = torch.empty(units, T, dtype=torch.float64, device=K.device)
    assert scores.is_contiguous() and scores.dtype == torch.float64
    _check(lib().nq_score_static(_ptr(K), kv_strides(K), units, heads, T, int(W), _ptr(scores),
                                 _stream(stream)))
    return scores


def nq_select(scores: torch.Tensor, W: int, evict_pct: int, kept: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """kept [units][n] int32 ascending positions (see nq.h, nq_select)."""
    _require_cuda(scores)
    units, T = scores.shape
    n = kept_count(T, W, evict_pct)
    if kept is None:
        kept = torch.empty(units, n, dtype=torch.int32, device=scores.device)
    assert kept.dtype == torch.int32 and kept.stride(1) == 1
    _check(lib().nq_select(_ptr(scores), units, T, int(W), int(evict_pct), _ptr(kept),
                           kept.stride(0), _stream(stream)))
    return kept


def nq_encode(K: torch.Tensor | None, V: torch.Tensor | None, k_out: PackedStore | None,
              v_out: PackedStore | None, n: int, rope_tab: torch.Tensor | None = None,
              rope_max_pos: int = 0, kept: torch.Tensor | None = None, pos_base: int = 0,
              slot0: int = 0, stream=None):
    """Encode n slots of every (unit, head) into the packed stores (see nq.h, nq_encode).
    K and V may also be pinned host tensors: the kernel then reads only the rows
    it encodes (the kept ones) across the bus."""
    _require_device_readable(K, V)
    _require_cuda(kept, rope_tab)
    ref = K if K is not None else V
    units, heads, T_in, _ = ref.shape
    kd = k_out.desc() if K is not None else None
    vd = v_out.desc() if V is not None else None
    ks = kv_strides(K) if K is not None else KVStrides(0, 0, 0)
    vs = kv_strides(V) if V is not None else KVStrides(0, 0, 0)
    if kept is not None:
        assert kept.dtype == torch.int32 and kept.stride(-1) == 1
    for st in (k_out if K is not None else None, v_out if V is not None else None):
        if st is not None and (st.meta.shape[0] < units or st.meta.shape[1] < heads
                               or st.meta.shape[2] < slot0 + n):
            raise ValueError("packed store too small for units x heads x (slot0 + n)")
    _check(lib().nq_encode(_ptr(K), ks, _ptr(V), vs, units, heads, T_in, int(n), _ptr(kept),
                           kept.stride(0) if kept is not None else 0, int(pos_base),
                           _ptr(rope_tab), int(rope_max_pos),
                           ctypes.byref(kd) if kd is not None else None,
                           ctypes.byref(vd) if vd is not None else None, int(slot0),
                           _stream(stream)))


def nq_decode(k_in: PackedStore | None, v_in: PackedStore | None, n: int,
              K_out: torch.Tensor | None, V_out: torch.Tensor | None,
              rope_tab: torch.Tensor | None = None, rope_max_pos: int = 0,
              positions: torch.Tensor | None = None, pos_base: int = 0, slot0: int = 0,
              stream=None):
    """Decode n slots of every (unit, head) into bf16 outputs (see nq.h, nq_decode)."""
    _require_cuda(K_out, V_out, positions, rope_tab)
    ref = K_out if K_out is not None else V_out
    units, heads = ref.shape[0], ref.shape[1]
    kd = k_in.desc() if K_out is not None else None
    vd = v_in.desc() if V_out is not None else None
    kos = kv_strides(K_out) if K_out is not None else KVStrides(0, 0, 0)
    vos = kv_strides(V_out) if V_out is not None else KVStrides(0, 0, 0)
    if positions is not None:
        assert positions.dtype == torch.int32 and positions.stride(-1) == 1
    for st in (k_in if K_out is not None else None, v_in if V_out is not None else None):
        if st is not None and (st.meta.shape[0] < units or st.meta.shape[1] < heads
                               or st.meta.shape[2] < slot0 + n):
            raise ValueError("packed store too small for units x heads x (slot0 + n)")
    for o in (K_out, V_out):
        if o is not None and o.shape[2] < n:
            raise ValueError("output has fewer than n tokens")
    _check(lib().nq_decode(ctypes.byref(kd) if kd is not None else None,
                           ctypes.byref(vd) if vd is not None else None, units, heads, int(n),
                           int(slot0), _ptr(positions),
                           positions.stride(0) if positions is not None else 0, int(pos_base),
                           _ptr(rope_tab), int(rope_max_pos), _ptr(K_out), kos, _ptr(V_out),
                           vos, _stream(stream)))


def nq_encode_exact(K: torch.Tensor | None, V: torch.Tensor | None, k_out: ExactStore | None,
                    v_out: ExactStore | None, n: int, rope_tab: torch.Tensor | None = None,
                    rope_max_pos: int = 0, kept: torch.Tensor | None = None, pos_base: int = 0,
                    slot0: int = 0, stream=None):
    """nq_encode into exact-layout stores (see nq.h, nq_encode_exact)."""
    _require_device_readable(K, V)
    _require_cuda(kept, rope_tab)
    ref = K if K is not None else V
    units, heads, T_in, _ = ref.shape
    kd = k_out.desc() if K is not None else None
    vd = v_out.desc() if V is not None else None
    ks = kv_strides(K) if K is not None else KVStrides(0, 0, 0)
    vs = kv_strides(V) if V is not None else KVStrides(0, 0, 0)
    if kept is not None:
        assert kept.dtype == torch.int32 and kept.stride(-1) == 1
    for st in (k_out if K is not None else None, v_out if V is not None else None):
        if st is not None and (st.sigma.shape[0] < units or st.sigma.shape[1] < heads
                               or st.sigma.shape[2] < slot0 + n):
            raise ValueError("exact store too small for units x heads x (slot0 + n)")
    _check(lib().nq_encode_exact(_ptr(K), ks, _ptr(V), vs, units, heads, T_in, int(n), _ptr(kept),
                                 kept.stride(0) if kept is not None else 0, int(pos_base),
                                 _ptr(rope_tab), int(rope_max_pos),
                                 ctypes.byref(kd) if kd is not None else None,
                                 ctypes.byref(vd) if vd is not None else None, int(slot0),
                                 _stream(stream)))


def nq_decode_exact(k_in: ExactStore | None, v_in: ExactStore | None, n: int,
                    K_out: torch.Tensor | None, V_out: torch.Tensor | None,
                    rope_tab: torch.Tensor | None = None, rope_max_pos: int = 0,
                    positions: torch.Tensor | None = None, pos_base: int = 0, slot0: int = 0,
                    stream=None):
    """nq_decode from exact-layout stores (see nq.h, nq_decode_exact)."""
    _require_cuda(K_out, V_out, positions, rope_tab)
    ref = K_out if K_out is not None else V_out
    units, heads = ref.shape[0], ref.shape[1]
    kd = k_in.desc() if K_out is not None else None
    vd = v_in.desc() if V_out is not None else None
    kos = kv_strides(K_out) if K_out is not None else KVStrides(0, 0, 0)
    vos = kv_strides(V_out) if V_out is not None else KVStrides(0, 0, 0)
    if positions is not None:
        assert positions.dtype == torch.int32 and positions.stride(-1) == 1
    for st in (k_in if K_out is not None else None, v_in if V_out is not None else None):
        if st is not None and (st.sigma.shape[0] < units or st.sigma.shape[1] < heads
                               or st.sigma.shape[2] < slot0 + n):
            raise ValueError("exact store too small for units x heads x (slot0 + n)")
    for o in (K_out, V_out):
        if o is not None and o.shape[2] < n:
            raise ValueError("output has fewer than n tokens")
    _check(lib().nq_decode_exact(ctypes.byref(kd) if kd is not None else None,
                                 ctypes.byref(vd) if vd is not None else None, units, heads,
                                 int(n), int(slot0), _ptr(positions),
                                 positions.stride(0) if positions is not None else 0,
                                 int(pos_base), _ptr(rope_tab), int(rope_max_pos), _ptr(K_out),
                                 kos, _ptr(V_out), vos, _stream(stream)))


def nq_attend(q: torch.Tensor, k_in: PackedStore, v_in: PackedStore, n: int, G: int,
              rope_tab: torch.Tensor, rope_max_pos: int, scale: float | None = None,
              positions: torch.Tensor | None = None, pos_base: int = 0, slot0: int = 0,
              ws: torch.Tensor | None = None, stream=None):
    """Decode-phase attention of q [units][heads*G][128] (fp32) over n packed
    slots per (unit, KV head): returns (out fp32 [units][heads*G][128],
    lse fp32 [units][heads*G]) (see nq.h, nq_attend)."""
    _require_cuda(q, positions, rope_tab)
    if q.dtype != torch.float32 or not q.is_contiguous() or q.dim() != 3 or q.shape[2] != 128:
        raise ValueError("q must be a contiguous float32 [units, heads*G, 128] tensor")
    units, Hq = q.shape[0], q.shape[1]
    heads = k_in.meta.shape[1]
    if Hq != heads * G:
        raise ValueError("q has %d heads, expected heads * G = %d" % (Hq, heads * G))
    if positions is not None:
        assert positions.dtype == torch.int32 and positions.stride(-1) == 1
    out = torch.empty(units, Hq, 128, dtype=torch.float32, device=q.device)
    lse = torch.empty(units, Hq, dtype=torch.float32, device=q.device)
    need = lib().nq_attend_workspace_bytes(units, heads, G, int(n))
    if ws is None or ws.numel() * ws.element_size() < need:
        ws = torch.empty(max(need, 16) // 4, dtype=torch.float32, device=q.device)
    kd, vd = k_in.desc(), v_in.desc()
    _check(lib().nq_attend(_ptr(q), units, heads, int(G), ctypes.byref(kd), ctypes.byref(vd),
                           int(n), int(slot0), _ptr(positions),
                           positions.stride(0) if positions is not None else 0, int(pos_base),
                           _ptr(rope_tab), int(rope_max_pos),
                           float(scale if scale is not None else 128 ** -0.5), _ptr(out),
                           _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return out, lse


def nq_e8_quantise(y: torch.Tensor, bits: int, stream=None):
    """E8 step alone on [groups][8] fp32 rows (device): returns (codes int32
    [groups], code k of a group at bits [bits*k, bits*k + bits); coset uint8
    [groups], 1 = half-integer coset)."""
    _require_cuda(y)
    if y.dtype != torch.float32 or y.dim() != 2 or y.shape[1] != 8 or not y.is_contiguous():
        raise ValueError("y must be a contiguous float32 [groups, 8] tensor")
    g = y.shape[0]
    codes = torch.empty(g, dtype=torch.int32, device=y.device)
    coset = torch.empty(g, dtype=torch.uint8, device=y.device)
    _check(lib().nq_e8_quantise(_ptr(y), g, int(bits), _ptr(codes), _ptr(coset), _stream(stream)))
    return codes, coset


def nq_e8_box_quantise(y: torch.Tensor, bits: int, stream=None):
    """The exact layout's lattice step alone on [groups][8] fp32 rows (device):
    returns (codes int32 [groups] with the coset bit in the low bit of code 7,
    coset uint8 [groups])."""
    _require_cuda(y)
    if y.dtype != torch.float32 or y.dim() != 2 or y.shape[1] != 8 or not y.is_contiguous():
        raise ValueError("y must be a contiguous float32 [groups, 8] tensor")
    g = y.shape[0]
    codes = torch.empty(g, dtype=torch.int32, device=y.device)
    coset = torch.empty(g, dtype=torch.uint8, device=y.device)
    _check(lib().nq_e8_box_quantise(_ptr(y), g, int(bits), _ptr(codes), _ptr(coset),
                                    _stream(stream)))
    return codes, coset


class EntropyCoded:
    """Output of nq_entropy_encode (device tensors; see nq.h): words (uint16 in
    an int16 tensor of capacity nq_entropy_max_words), offsets (uint32 in an
    int32 tensor, [streams + 1]) and freq ([units][heads][2^bits], uint16 in
    int16)."""

    def __init__(self, words, offsets, freq, units, heads, n, bits, delta):
        self.words, self.offsets, self.freq = words, offsets, freq
        self.units, self.heads, self.n, self.bits, self.delta = units, heads, n, bits, delta

    def total_words(self) -> int:
        """Coded length in 16-bit words (reads offsets[streams]: synchronises)."""
        return int(self.offsets[-1].item()) & 0xFFFFFFFF

    def coded_bytes(self) -> int:
        """Stream words plus offsets and tables, as stored."""
        return 2 * self.total_words() + 4 * self.offsets.numel() + 2 * self.freq.numel()


def entropy_workspace(units: int, heads: int, n: int, device="cuda") -> torch.Tensor:
    need = lib().nq_entropy_workspace_bytes(units, heads, int(n))
    return torch.empty(max(need, 16) // 4 + 4, dtype=torch.int32, device=device)


def nq_entropy_encode(store: PackedStore, n: int, delta: bool = True, slot0: int = 0,
                      ws: torch.Tensor | None = None, coded: EntropyCoded | None = None,
                      stream=None) -> EntropyCoded:
    """Delta + rANS coding of the codes of slots slot0 .. slot0+n-1 of every
    (unit, head) of a packed store (see nq.h, nq_entropy_encode).  ws and
    coded (a previous result of the same shape) may be given to reuse memory."""
    _require_cuda(store.codes)
    units, heads = store.meta.shape[0], store.meta.shape[1]
    dev = store.codes.device
    L = lib()
    S = L.nq_entropy_streams(units, heads, int(n))
    cap = L.nq_entropy_max_words(units, heads, int(n))
    need = L.nq_entropy_workspace_bytes(units, heads, int(n))
    if (coded is not None and coded.words.numel() >= cap and coded.offsets.numel() == S + 1
            and tuple(coded.freq.shape) == (units, heads, 1 << store.bits)):
        words, offsets, freq = coded.words, coded.offsets, coded.freq
    else:
        words = torch.empty(max(cap, 1), dtype=torch.int16, device=dev)
        offsets = torch.empty(S + 1, dtype=torch.int32, device=dev)
        freq = torch.empty(units, heads, 1 << store.bits, dtype=torch.int16, device=dev)
    if ws is None or ws.numel() * ws.element_size() < need:
        ws = entropy_workspace(units, heads, n, dev)
    d = store.desc()
    _check(L.nq_entropy_encode(ctypes.byref(d), units, heads, int(n), int(slot0), int(delta),
                               _ptr(freq), _ptr(offsets), _ptr(words), cap, _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)))
    return EntropyCoded(words, offsets, freq, units, heads, int(n), store.bits, bool(delta))


def nq_entropy_decode(coded: EntropyCoded, out: PackedStore, slot0: int = 0, stream=None):
    """Write the codes of slots slot0 .. slot0+n-1 of `out` from an
    EntropyCoded (meta untouched; see nq.h, nq_entropy_decode)."""
    _require_cuda(out.codes, coded.words)
    if out.bits != coded.bits or out.meta.shape[0] != coded.units or out.meta.shape[1] != coded.heads:
        raise ValueError("output store does not match the coded shape / bits")
    d = out.desc()
    _check(lib().nq_entropy_decode(_ptr(coded.words), _ptr(coded.offsets), _ptr(coded.freq),
                                   coded.units, coded.heads, coded.n, int(coded.delta),
                                   ctypes.byref(d), int(slot0), _stream(stream)))


DECODE_AUTO, DECODE_TENSOR_CORES, DECODE_CUDA_CORES = 0, 1, 2


def set_decode_engine(engine: int) -> None:
    """Select the decode kernel (nq.h, nq_set_decode_engine); process-wide."""
    _check(lib().nq_set_decode_engine(int(engine)))


def get_decode_engine() -> int:
    return int(lib().nq_get_decode_engine())


def device_error() -> int:
    v = ctypes.c_uint32(0)
    _check(lib().nq_device_error(ctypes.byref(v)))
    return int(v.value)


# ------------------------------------------------------- whole-cache helper
class Codec:
    """One layer-batched compression pass (score -> select -> encode) and its
    inverse, all through the C ABI.  Buffers are allocated once per shape."""

    def __init__(self, units: int, heads: int, T: int, theta: float, bits_k: int = 3,
                 bits_v: int = 2, window: int = 64, evict_pct: int = 0, device="cuda",
                 max_pos: int | None = None):
        self.units, self.heads, self.T = units, heads, T
        self.W, self.pct = window, evict_pct
        self.bits_k, self.bits_v = bits_k, bits_v
        self.evict = evict_pct > 0 and T > 1 + window
        self.n = kept_count(T, window, evict_pct) if self.evict else T
        self.max_pos = max_pos or T
        self.rope = rope_tables(theta, self.max_pos, device)
        self.k_store = PackedStore.empty(units, heads, self.n, bits_k, device)
        self.v_store = PackedStore.empty(units, heads, self.n, bits_v, device)
        if self.evict:
            self.scores = torch.empty(units, T, dtype=torch.float64, device=device)
            self.ws = score_workspace(units, heads, device)
            self.kept = torch.empty(units, self.n, dtype=torch.int32, device=device)
        else:
            self.kept = None

    def encode(self, K: torch.Tensor, V: torch.Tensor, stream=None, units: slice | None = None):
        """Compress K, V [units][heads][T][128]; with `units`, only that range
        of units (K and V are then the full-cache tensors)."""
        u = units or slice(0, self.units)
        kept = self.kept[u] if self.kept is not None else None
        if self.evict:
            ws = self.ws.view(self.units, -1)[u] if self.ws.numel() % self.units == 0 else self.ws
            nq_score(K[u] if units else K, self.W, self.scores[u], ws, stream)
            nq_select(self.scores[u], self.W, self.pct, kept, stream)
        nq_encode(K[u] if units else K, V[u] if units else V, self.k_store.select_units(u),
                  self.v_store.select_units(u), self.n, self.rope, self.max_pos, kept=kept,
                  stream=stream)

    def decode(self, K_out: torch.Tensor, V_out: torch.Tensor, stream=None,
               units: slice | None = None):
        u = units or slice(0, self.units)
        nq_decode(self.k_store.select_units(u), self.v_store.select_units(u), self.n,
                  K_out[u] if units else K_out, V_out[u] if units else V_out, self.rope,
                  self.max_pos, positions=self.kept[u] if self.kept is not None else None,
                  stream=stream)

    @property
    def packed_bytes(self) -> int:
        b = self.k_store.nbytes + self.v_store.nbytes
        if self.kept is not None:
            b += self.kept.numel() * 4
        return b


class HostRoundTrip:
    """Compress a cache that lives in pinned host memory and write its
    reconstruction back to pinned host memory, in chunks of units (one by
    default: the finest pipeline measured fastest) on three streams: the
    host-to-device copy of chunk c+1, the kernels of chunk c and the
    device-to-host copy of chunk c-1 run at the same time (the two copy
    directions share nothing on a full-duplex link).  The device tensors are
    the codec's working copies; every run() is asynchronous on the caller's
    current stream, which afterwards waits for the last copy.

    Host tensors with fewer units than the run (R of them) act as a ring: unit
    u is copied from and to host slot u % R, every unit still crossing the bus
    both ways (for hosts that cannot pin a whole cache; values must then be
    copied, not read in place, and R must be a multiple of the chunk)."""

    def __init__(self, codec: Codec, K: torch.Tensor, V: torch.Tensor, K_out: torch.Tensor,
                 V_out: torch.Tensor, chunk_units: int = 1, values_in_place: bool | None = None,
                 units: int | None = None):
        self.codec, self.K, self.V, self.K_out, self.V_out = codec, K, V, K_out, V_out
        # With eviction only the kept value rows are needed: the encode kernel
        # reads them straight from the pinned host cache, so the rows it drops
        # never cross the bus (keys are copied whole: every key is scored).
        self.values_in_place = codec.evict if values_in_place is None else values_in_place
        # the leading `units` units of the codec (all by default)
        self.units = codec.units if units is None else min(int(units), codec.units)
        self.chunks = [slice(u, min(u + chunk_units, self.units))
                       for u in range(0, self.units, chunk_units)]
        self.h2d, self.comp, self.d2h = (torch.cuda.Stream(K.device) for _ in range(3))
        ev = lambda: [torch.cuda.Event() for _ in self.chunks]  # noqa: E731
        self.in_ready, self.comp_done, self.out_done = ev(), ev(), ev()
        self.ran = False

    def h2d_bytes(self, Kh: torch.Tensor, Vh: torch.Tensor) -> int:
        """Bytes that cross the bus host-to-device per run."""
        per_unit = lambda t: t[0].numel() * t.element_size()  # noqa: E731
        if not self.values_in_place:
            return self.units * (per_unit(Kh) + per_unit(Vh))
        c = self.codec
        return self.units * (per_unit(Kh) + c.heads * c.n * 128 * Vh.element_size())

    def d2h_bytes(self, K_out_h: torch.Tensor, V_out_h: torch.Tensor) -> int:
        """Bytes that cross the bus device-to-host per run."""
        return self.units * (K_out_h[0].numel() * K_out_h.element_size()
                             + V_out_h[0].numel() * V_out_h.element_size())

    def run(self, Kh: torch.Tensor, Vh: torch.Tensor, K_out_h: torch.Tensor,
            V_out_h: torch.Tensor):
        R = Kh.shape[0]
        if R < self.units:
            step = self.chunks[0].stop - self.chunks[0].start
            if self.values_in_place or R % step or min(Vh.shape[0], K_out_h.shape[0],
                                                       V_out_h.shape[0]) < R:
                raise ValueError("a host ring needs copied values, equal ring sizes and a "
                                 "multiple of the chunk")

        def host(u: slice) -> slice:  # the host slot of a chunk
            return u if R >= self.units else slice(u.start % R, u.start % R + u.stop - u.start)

        caller = torch.cuda.current_stream(self.K.device)
        start = torch.cuda.Event()
        start.record(caller)
        for s in (self.h2d, self.comp, self.d2h):
            s.wait_event(start)
        for c, u in enumerate(self.chunks):
            with torch.cuda.stream(self.h2d):
                if self.ran:  # the previous run's kernels are done reading this chunk
                    self.h2d.wait_event(self.comp_done[c])
                self.K[u].copy_(Kh[host(u)], non_blocking=True)
                if not self.values_in_place:
                    self.V[u].copy_(Vh[host(u)], non_blocking=True)
                self.in_ready[c].record(self.h2d)
            self.comp.wait_event(self.in_ready[c])
            if self.ran:  # the previous run's copy-out of this chunk is done
                self.comp.wait_event(self.out_done[c])
            self.codec.encode(self.K, Vh if self.values_in_place else self.V, self.comp, units=u)
            self.codec.decode(self.K_out, self.V_out, self.comp, units=u)
            self.comp_done[c].record(self.comp)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(self.comp_done[c])
                K_out_h[host(u)].copy_(self.K_out[u], non_blocking=True)
                V_out_h[host(u)].copy_(self.V_out[u], non_blocking=True)
                self.out_done[c].record(self.d2h)
        caller.wait_event(self.out_done[-1])
        self.ran = True


# ------------------------------------------------------- whole-cache pipelines
class LayeredCache:
    """A model's cache [layers][heads][T][128] compressed layer-batched, with
    boundary layers kept in bf16 (NexusQuant "Implementation details":
    protect_boundary keeps the first/last layers at full precision).

    The quantised layers must form one contiguous range (they do for
    protect_boundary).  Protected layers pass through as a bf16 device copy;
    every quantised layer runs score -> select -> encode through the C ABI."""

    def __init__(self, layers: int, heads: int, T: int, theta: float, bits_k: int = 3,
                 bits_v: int = 2, window: int = 64, evict_pct: int = 0,
                 protected: tuple = (), device="cuda"):
        q = [l for l in range(layers) if l not in set(protected)]
        if q and q != list(range(q[0], q[-1] + 1)):
            raise ValueError("quantised layers must be contiguous")
        self.layers, self.q0, self.q1 = layers, (q[0] if q else 0), (q[-1] + 1 if q else 0)
        self.protected = tuple(sorted(set(protected)))
        self.codec = Codec(self.q1 - self.q0, heads, T, theta, bits_k, bits_v, window, evict_pct,
                           device) if q else None
        self.kept_bf16_K = {}
        self.kept_bf16_V = {}

    def encode(self, K: torch.Tensor, V: torch.Tensor, stream=None):
        for l in self.protected:
            self.kept_bf16_K[l] = K[l].clone()
            self.kept_bf16_V[l] = V[l].clone()
        if self.codec is not None:
            self.codec.encode(K[self.q0:self.q1], V[self.q0:self.q1], stream)

    def decode_quantised(self, K_out: torch.Tensor, V_out: torch.Tensor, stream=None):
        """Reconstruct the quantised layers into [q1-q0][heads][n][128] outputs."""
        self.codec.decode(K_out, V_out, stream)

    @property
    def stored_bits(self) -> int:
        b = 0 if self.codec is None else self.codec.packed_bytes * 8
        for l in self.protected:
            b += 16 * (self.kept_bf16_K[l].numel() + self.kept_bf16_V[l].numel()) if l in self.kept_bf16_K else 0
        return b


class AppendStore:
    """Packed caches of many sequences x layers with room to append tokens
    (the decode-append regime): units = sequences * layers, slot capacity cap.
    append() encodes one new token per unit at its position (slot = position);
    decode_layer() reconstructs all tokens of one layer for every sequence."""

    def __init__(self, sequences: int, layers: int, heads: int, cap: int, theta: float,
                 bits_k: int = 2, bits_v: int = 2, device="cuda"):
        self.S, self.L, self.H, self.cap = sequences, layers, heads, cap
        self.bits_k, self.bits_v = bits_k, bits_v
        self.rope = rope_tables(theta, cap, device)
        self.k = PackedStore.empty(sequences * layers, heads, cap, bits_k, device)
        self.v = PackedStore.empty(sequences * layers, heads, cap, bits_v, device)

    def _units(self, store: PackedStore, seq: int | None = None, layer: int | None = None):
        c = store.codes.view(self.S, self.L, self.H, self.cap, -1)
        m = store.meta.view(self.S, self.L, self.H, self.cap)
        if seq is not None:
            c, m = c[seq:seq + 1], m[seq:seq + 1]
        if layer is not None:
            c, m = c[:, layer], m[:, layer]
        else:
            c, m = c.reshape(-1, self.H, self.cap, c.shape[-1]), m.reshape(-1, self.H, self.cap)
        return PackedStore(c, m, store.bits)

    def fill(self, seq: int, K: torch.Tensor, V: torch.Tensor, stream=None):
        """Encode an initial cache [layers][heads][T0][128] of one sequence at positions 0..T0-1."""
        n = K.shape[2]
        nq_encode(K, V, self._units(self.k, seq), self._units(self.v, seq), n, self.rope, self.cap,
                  stream=stream)

    def append(self, K_new: torch.Tensor, V_new: torch.Tensor, pos: int, stream=None):
        """K_new/V_new [sequences*layers][heads][1][128]: one token per unit at position pos."""
        nq_encode(K_new, V_new, self.k, self.v, 1, self.rope, self.cap, pos_base=pos, slot0=pos,
                  stream=stream)

    def decode_layer(self, layer: int, n: int, K_out: torch.Tensor, V_out: torch.Tensor,
                     stream=None):
        """Slots 0..n-1 of `layer` for every sequence into [sequences][heads][n][128]."""
        nq_decode(self._units(self.k, layer=layer), self._units(self.v, layer=layer), n, K_out,
                  V_out, self.rope, self.cap, stream=stream)
