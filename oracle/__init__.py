"""CPU oracle of the KV-cache eviction + E8 lattice quantisation hot path.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product path (the
CUDA library and its binding) never calls it.

The arithmetic lives in ``nq_oracle.c`` (plain C, fp32 with explicit fmaf,
-ffp-contract=off); this module compiles it with gcc on first use and wraps it
with numpy marshalling.  Every function cites, in the C source, the passage of
the method description it follows:

* "NexusQuant: training-free 10-33x KV cache compression" (zingnex.cn),
  sections "Token eviction", "E8 lattice quantisation", "Implementation
  details";
* "Como comprimir o KV cache do seu LLM em 33x sem treino" (dev.to), section
  "Como funciona (em 6 passos)", steps 1-6.

Parity unpinned: end-to-end model quality (perplexity) -- it needs trained
models and datasets.  Every other function is pinned by ``tests/test_oracle_*``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboq.so")
_lock = threading.Lock()
_lib = None

D = 128

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile nq_oracle.c into _build/liboq.so (gcc); returns the path."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_SO)) or os.path.getmtime(_SO) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        # NQ_ORACLE_SO points the tests that plant mistakes at a mutated build
        lib = ctypes.CDLL(os.environ.get("NQ_ORACLE_SO") or build())
        P = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        sig = {
            "oq_score": (None, [P, i32, i32, i32, P, P]),
            "oq_kept_count": (i64, [i64, i64, i32]),
            "oq_select": (i64, [P, i64, i64, i32, P]),
            "oq_encode_unit": (i64, [P, P, i32, i64, i64, P, i64, dbl, i32, i32, P, P, P, P]),
            "oq_decode_unit": (None, [P, P, P, P, i32, i64, P, i64, dbl, i32, i32, P, P]),
            "oq_e8_batch": (None, [P, i64, P, P, P]),
            "oq_e8_code_batch": (None, [P, i64, ctypes.c_int, P, P]),
            "oq_reconstruct_batch": (None, [P, P, i64, ctypes.c_int, P, P, ctypes.c_int, P]),
            "oq_attend_unit": (None, [P, P, P, P, ctypes.c_int, ctypes.c_int, i64, P, i64,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_int, P,
                                      ctypes.c_double, P, P]),
            "oq_fwht_batch": (None, [P, i64]),
            "oq_f32_to_f16_batch": (None, [P, i64, P]),
            "oq_f32_to_bf16_batch": (None, [P, i64, P]),
            "oq_rope_batch": (None, [dbl, P, i64, P, P]),
            "oq_rope_apply_batch": (None, [P, P, P, i64, i32]),
            "oq_encode_batch": (i64, [P, i64, i32, P, P, i32, P, P]),
            "oq_decode_batch": (None, [P, P, i64, i32, P, P, i32, P]),
            "oq_e8_box_code_batch": (None, [P, i64, i32, P, P, P]),
            "oq_encode_box_batch": (i64, [P, i64, i32, P, P, i32, P, P]),
            "oq_fold_exact_batch": (None, [P, P, i64, i32, P, P]),
            "oq_unfold_exact_batch": (None, [P, P, i64, i32, P, P]),
            "oq_encode_margin_batch": (None, [P, i64, i32, P, P, i32, P]),
            "oq_e8_margin_batch": (None, [P, i64, P]),
            "oq_exact_pack_group": (ctypes.c_uint32, [P, i32, i32]),
            "oq_exact_unpack_group": (None, [ctypes.c_uint32, i32, P, P]),
            "oq_ans_table": (None, [P, i32, P]),
            "oq_ans_encode": (i64, [P, i64, P, i32, P, i64]),
            "oq_ans_decode": (i64, [P, i64, P, i32, P, i64]),
            "oq_entropy_encode_store": (i64, [P, i64, i32, i64, i32, i32, P, P, P, i64]),
            "oq_entropy_decode_store": (i32, [P, P, P, i64, i32, i64, i32, i32, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _u16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.uint16:
        a = a.view(np.uint16) if a.dtype.itemsize == 2 else a.astype(np.uint16)
    return np.ascontiguousarray(a)


# ---------------------------------------------------------------- scalars
def f32_to_f16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.empty(x.size, np.uint16)
    _load().oq_f32_to_f16_batch(_p(x), x.size, _p(out))
    return out


def f32_to_bf16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.empty(x.size, np.uint16)
    _load().oq_f32_to_bf16_batch(_p(x), x.size, _p(out))
    return out


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------- transforms
def fwht(v) -> np.ndarray:
    """Unnormalised Sylvester FWHT of [..., 128] fp32 rows (stages h ascending)."""
    v = np.array(v, dtype=np.float32, copy=True, order="C")
    shp = v.shape
    v = v.reshape(-1, D)
    _load().oq_fwht_batch(_p(v), v.shape[0])
    return v.reshape(shp)


def rope_cs(theta: float, pos) -> tuple[np.ndarray, np.ndarray]:
    """fp32 (cos, sin) rows [n][64] for the given positions (two-level rule)."""
    pos = np.ascontiguousarray(np.atleast_1d(pos), dtype=np.int64)
    c = np.empty((pos.size, D // 2), np.float32)
    s = np.empty((pos.size, D // 2), np.float32)
    _load().oq_rope_batch(float(theta), _p(pos), pos.size, _p(c), _p(s))
    return c, s


def rope_apply(v, c, s, direction: int) -> np.ndarray:
    """direction -1: undo (rotate by -angle); +1: redo.  v [n][128] fp32."""
    v = np.array(v, dtype=np.float32, copy=True, order="C").reshape(-1, D)
    c = np.ascontiguousarray(c, dtype=np.float32).reshape(-1, D // 2)
    s = np.ascontiguousarray(s, dtype=np.float32).reshape(-1, D // 2)
    _load().oq_rope_apply_batch(_p(v), _p(c), _p(s), v.shape[0], int(direction))
    return v


def e8_nearest(y) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Nearest E8 point of [n][8] fp32 groups.

    Returns (t = 2q int32 [n][8], coset int32 [n] (1 = half-integer), fp32 distance [n])."""
    y = np.ascontiguousarray(y, dtype=np.float32).reshape(-1, 8)
    n = y.shape[0]
    t = np.empty((n, 8), np.int32)
    cs = np.empty(n, np.int32)
    d = np.empty(n, np.float32)
    _load().oq_e8_batch(_p(y), n, _p(t), _p(cs), _p(d))
    return t, cs, d


def e8_codes(y, bits: int) -> tuple[np.ndarray, np.ndarray]:
    """E8 step with codes of [n][8] fp32 groups: (codes uint32 [n], code k of a
    group at bits [bits*k, bits*k + bits); coset int32 [n])."""
    y = np.ascontiguousarray(y, dtype=np.float32).reshape(-1, 8)
    n = y.shape[0]
    codes = np.empty(n, np.uint32)
    cs = np.empty(n, np.int32)
    _load().oq_e8_code_batch(_p(y), n, int(bits), _p(codes), _p(cs))
    return codes, cs


# ------------------------------------------------------ vector codec
def words_per_vector(bits: int) -> int:
    return 4 * bits


def encode_vectors(x_bf16, bits: int, rope: bool = False, c=None, s=None):
    """Encode [n][128] bf16 vectors; returns (words [n][4b] u32, meta [n] u32, clamps)."""
    x = _u16(x_bf16).reshape(-1, D)
    n = x.shape[0]
    if c is None:
        c = np.zeros((n, D // 2), np.float32)
        s = np.zeros((n, D // 2), np.float32)
    c = np.ascontiguousarray(c, dtype=np.float32).reshape(n, D // 2)
    s = np.ascontiguousarray(s, dtype=np.float32).reshape(n, D // 2)
    w = np.empty((n, 4 * bits), np.uint32)
    m = np.empty(n, np.uint32)
    cl = _load().oq_encode_batch(_p(x), n, int(rope), _p(c), _p(s), bits, _p(w), _p(m))
    return w, m, int(cl)


def encode_margins(x_bf16, bits: int, rope: bool = False, c=None, s=None) -> np.ndarray:
    """Per vector, the smallest relative distance of any encode decision to
    its boundary (0 on a boundary, at most 1): the scale's fp16 rounding, each
    coordinate's rounding, the parity move and the coset choice.  Used to tell
    excusable GPU/oracle mismatches (near a boundary) from real ones."""
    x = _u16(x_bf16).reshape(-1, D)
    n = x.shape[0]
    if c is None:
        c = np.zeros((n, D // 2), np.float32)
        s = np.zeros((n, D // 2), np.float32)
    c = np.ascontiguousarray(c, dtype=np.float32).reshape(n, D // 2)
    s = np.ascontiguousarray(s, dtype=np.float32).reshape(n, D // 2)
    out = np.empty(n, np.float64)
    _load().oq_encode_margin_batch(_p(x), n, int(rope), _p(c), _p(s), bits, _p(out))
    return out


def e8_margins(y) -> np.ndarray:
    """Per group of 8 fp32 coordinates, the smallest relative distance of an
    E8 decision (rounding, parity move, coset choice) to its boundary."""
    y = np.ascontiguousarray(y, dtype=np.float32).reshape(-1, 8)
    out = np.empty(y.shape[0], np.float64)
    _load().oq_e8_margin_batch(_p(y), y.shape[0], _p(out))
    return out


def decode_vectors(words, meta, bits: int, rope: bool = False, c=None, s=None):
    """Decode [n] packed vectors to [n][128] bf16 bits (uint16)."""
    words = np.ascontiguousarray(words, dtype=np.uint32).reshape(-1, 4 * bits)
    meta = np.ascontiguousarray(meta, dtype=np.uint32).ravel()
    n = words.shape[0]
    if c is None:
        c = np.zeros((n, D // 2), np.float32)
        s = np.zeros((n, D // 2), np.float32)
    c = np.ascontiguousarray(c, dtype=np.float32).reshape(n, D // 2)
    s = np.ascontiguousarray(s, dtype=np.float32).reshape(n, D // 2)
    out = np.empty((n, D), np.uint16)
    _load().oq_decode_batch(_p(words), _p(meta), n, int(rope), _p(c), _p(s), bits, _p(out))
    return out


def reconstruct_vectors(words, meta, bits: int, rope: bool = False, c=None, s=None):
    """fp32 reconstructions [n][128] of [n] packed vectors (the decode output
    before its bf16 rounding)."""
    words = np.ascontiguousarray(words, dtype=np.uint32).reshape(-1, 4 * bits)
    meta = np.ascontiguousarray(meta, dtype=np.uint32).ravel()
    n = words.shape[0]
    if c is None:
        c = np.zeros((n, D // 2), np.float32)
        s = np.zeros((n, D // 2), np.float32)
    c = np.ascontiguousarray(c, dtype=np.float32).reshape(n, D // 2)
    s = np.ascontiguousarray(s, dtype=np.float32).reshape(n, D // 2)
    out = np.empty((n, D), np.float32)
    _load().oq_reconstruct_batch(_p(words), _p(meta), n, int(rope), _p(c), _p(s), bits, _p(out))
    return out


# ------------------------------------------------------ unit level
def score_unit(K_unit, W: int, return_mean: bool = False):
    """Key-key proxy scores of one layer; K_unit [H][T][128] bf16."""
    K = _u16(K_unit)
    H, T, d = K.shape
    assert d == D
    out = np.empty(T, np.float64)
    mean = np.empty((H, D), np.float32)
    _load().oq_score(_p(K), H, T, int(W), _p(out), _p(mean))
    return (out, mean) if return_mean else out


def kept_count(T: int, W: int, pct: int) -> int:
    return int(_load().oq_kept_count(int(T), int(W), int(pct)))


def select(scores, W: int, pct: int) -> np.ndarray:
    """Ascending kept positions of one layer (int32)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    T = s.size
    kept = np.empty(T, np.int32)
    n = _load().oq_select(_p(s), T, int(W), int(pct), _p(kept))
    return kept[:n].copy()


def encode_unit(K_unit, V_unit, n: int, kept=None, pos_base: int = 0, theta: float = 1e4,
                bits_k: int = 3, bits_v: int = 2):
    """Encode one layer.  K_unit/V_unit [H][T_in][128] bf16 (or None).

    Returns dict with k_codes [H][n][4bk], k_meta [H][n], v_codes, v_meta, clamps."""
    K = _u16(K_unit) if K_unit is not None else None
    V = _u16(V_unit) if V_unit is not None else None
    ref = K if K is not None else V
    H, T_in, _ = ref.shape
    kp = None if kept is None else np.ascontiguousarray(kept, dtype=np.int32)
    kc = np.zeros((H, n, 4 * bits_k), np.uint32) if K is not None else None
    km = np.zeros((H, n), np.uint32) if K is not None else None
    vc = np.zeros((H, n, 4 * bits_v), np.uint32) if V is not None else None
    vm = np.zeros((H, n), np.uint32) if V is not None else None
    cl = _load().oq_encode_unit(_p(K), _p(V), H, T_in, n, _p(kp), int(pos_base), float(theta),
                                bits_k, bits_v, _p(kc), _p(km), _p(vc), _p(vm))
    return {"k_codes": kc, "k_meta": km, "v_codes": vc, "v_meta": vm, "clamps": int(cl)}


def decode_unit(k_codes, k_meta, v_codes, v_meta, positions=None, pos_base: int = 0,
                theta: float = 1e4, bits_k: int = 3, bits_v: int = 2):
    """Decode one layer to (K_out, V_out) [H][n][128] bf16 bits (or None)."""
    kc = None if k_codes is None else np.ascontiguousarray(k_codes, dtype=np.uint32)
    km = None if k_meta is None else np.ascontiguousarray(k_meta, dtype=np.uint32)
    vc = None if v_codes is None else np.ascontiguousarray(v_codes, dtype=np.uint32)
    vm = None if v_meta is None else np.ascontiguousarray(v_meta, dtype=np.uint32)
    ref = km if km is not None else vm
    H, n = ref.shape
    pp = None if positions is None else np.ascontiguousarray(positions, dtype=np.int32)
    Ko = np.empty((H, n, D), np.uint16) if kc is not None else None
    Vo = np.empty((H, n, D), np.uint16) if vc is not None else None
    _load().oq_decode_unit(_p(kc), _p(km), _p(vc), _p(vm), H, n, _p(pp), int(pos_base),
                           float(theta), bits_k, bits_v, _p(Ko), _p(Vo))
    return Ko, Vo


def attend_unit(k_codes, k_meta, v_codes, v_meta, q, G: int, scale: float, positions=None,
                pos_base: int = 0, theta: float = 1e4, bits_k: int = 3, bits_v: int = 2):
    """Decode-phase attention of q [H*G][128] (fp32) over one packed unit
    ([H][n] vectors): returns (out fp64 [H*G][128], lse fp64 [H*G])."""
    kc = np.ascontiguousarray(k_codes, dtype=np.uint32)
    km = np.ascontiguousarray(k_meta, dtype=np.uint32)
    vc = np.ascontiguousarray(v_codes, dtype=np.uint32)
    vm = np.ascontiguousarray(v_meta, dtype=np.uint32)
    H, n = km.shape
    q = np.ascontiguousarray(q, dtype=np.float32).reshape(H * G, D)
    pp = None if positions is None else np.ascontiguousarray(positions, dtype=np.int32)
    out = np.empty((H * G, D), np.float64)
    lse = np.empty(H * G, np.float64)
    _load().oq_attend_unit(_p(kc), _p(km), _p(vc), _p(vm), H, G, n, _p(pp), int(pos_base),
                           float(theta), bits_k, bits_v, _p(q), float(scale), _p(out), _p(lse))
    return out, lse


# ------------------------------------------------- delta + entropy stage
ANS_M = 4096
ANS_SEG = 2048  # tokens per stream segment


def ans_table(counts) -> np.ndarray:
    """Quantised rANS frequencies (sum 4096) of symbol counts."""
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    F = np.empty(counts.size, np.uint16)
    _load().oq_ans_table(_p(counts), counts.size, _p(F))
    return F


def ans_encode(sym, F) -> np.ndarray:
    """One rANS stream of 16-bit words (final state first)."""
    sym = np.ascontiguousarray(sym, dtype=np.uint8)
    F = np.ascontiguousarray(F, dtype=np.uint16)
    cap = sym.size + 2
    out = np.empty(cap, np.uint16)
    n = _load().oq_ans_encode(_p(sym), sym.size, _p(F), F.size, _p(out), cap)
    if n < 0:
        raise ValueError("oq_ans_encode failed (%d)" % n)
    return out[:n].copy()


def ans_decode(words, F, count: int) -> tuple[np.ndarray, int]:
    """Decode count symbols; returns (symbols, words read or -1)."""
    words = np.ascontiguousarray(words, dtype=np.uint16)
    F = np.ascontiguousarray(F, dtype=np.uint16)
    sym = np.empty(count, np.uint8)
    used = _load().oq_ans_decode(_p(words), words.size, _p(F), F.size, _p(sym), count)
    return sym, int(used)


def entropy_streams(units: int, heads: int, n: int) -> int:
    return units * heads * ((n + ANS_SEG - 1) // ANS_SEG) * D


def entropy_encode_store(codes, bits: int, delta: bool):
    """codes: uint32 [units][heads][n][4*bits].  Returns (freq [units][heads][2^bits]
    uint16, offsets [streams + 1] uint32, words uint16)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    units, heads, n = codes.shape[:3]
    S = entropy_streams(units, heads, n)
    cap = S * (ANS_SEG + 2)
    freq = np.empty((units, heads, 1 << bits), np.uint16)
    offsets = np.empty(S + 1, np.uint32)
    words = np.empty(cap, np.uint16)
    tot = _load().oq_entropy_encode_store(_p(codes), units, heads, n, bits, int(delta), _p(freq),
                                          _p(offsets), _p(words), cap)
    if tot < 0:
        raise ValueError("oq_entropy_encode_store failed")
    return freq, offsets, words[:tot].copy()


def entropy_decode_store(words, offsets, freq, units: int, heads: int, n: int, bits: int,
                         delta: bool) -> np.ndarray:
    """Inverse of entropy_encode_store: uint32 codes [units][heads][n][4*bits]."""
    words = np.ascontiguousarray(words, dtype=np.uint16)
    offsets = np.ascontiguousarray(offsets, dtype=np.uint32)
    freq = np.ascontiguousarray(freq, dtype=np.uint16)
    codes = np.empty((units, heads, n, 4 * bits), np.uint32)
    rc = _load().oq_entropy_decode_store(_p(words), _p(offsets), _p(freq), units, heads, n, bits,
                                         int(delta), _p(codes))
    if rc != 0:
        raise ValueError("oq_entropy_decode_store: inconsistent stream")
    return codes


# ------------------------------------------- E8 within the code box (exact packing)
def e8_box_codes(y, bits: int):
    """Box-constrained nearest E8 points of [n][8] fp32 groups: (codes uint32
    [n] with code i at bits [b i, b i + b), coset int32 [n], distance fp32 [n])."""
    y = np.ascontiguousarray(y, dtype=np.float32).reshape(-1, 8)
    n = y.shape[0]
    codes = np.empty(n, np.uint32)
    coset = np.empty(n, np.int32)
    dist = np.empty(n, np.float32)
    _load().oq_e8_box_code_batch(_p(y), n, bits, _p(codes), _p(coset), _p(dist))
    return codes, coset, dist


def exact_pack(j8, half: int, bits: int) -> int:
    """One group's 8 codes and coset bit in 8*bits bits (coset in the low bit of j_7)."""
    j = np.ascontiguousarray(j8, dtype=np.uint32)
    return int(_load().oq_exact_pack_group(_p(j), int(half), bits))


def exact_unpack(w: int, bits: int):
    """Inverse of exact_pack: (codes uint32 [8], coset)."""
    j = np.empty(8, np.uint32)
    h = ctypes.c_int(0)
    _load().oq_exact_unpack_group(ctypes.c_uint32(w), bits, _p(j), ctypes.byref(h))
    return j, h.value


def encode_vectors_box(x_bf16, bits: int, rope: bool = False, c=None, s=None):
    """Encode [n][128] bf16 vectors with the box-constrained E8 step (regular
    layout); returns (words [n][4b] u32, meta [n] u32)."""
    x = _u16(x_bf16).reshape(-1, D)
    n = x.shape[0]
    if c is None:
        c = np.zeros((n, D // 2), np.float32)
        s = np.zeros((n, D // 2), np.float32)
    c = np.ascontiguousarray(c, dtype=np.float32).reshape(n, D // 2)
    s = np.ascontiguousarray(s, dtype=np.float32).reshape(n, D // 2)
    w = np.empty((n, 4 * bits), np.uint32)
    m = np.empty(n, np.uint32)
    _load().oq_encode_box_batch(_p(x), n, int(rope), _p(c), _p(s), bits, _p(w), _p(m))
    return w, m


def fold_exact(words, meta, bits: int):
    """Regular layout -> exact layout: (words [n][4b] u32, sigma [n] u16)."""
    words = np.ascontiguousarray(words, dtype=np.uint32).reshape(-1, 4 * bits)
    meta = np.ascontiguousarray(meta, dtype=np.uint32).ravel()
    n = words.shape[0]
    out = np.empty_like(words)
    sig = np.empty(n, np.uint16)
    _load().oq_fold_exact_batch(_p(words), _p(meta), n, bits, _p(out), _p(sig))
    return out, sig


def unfold_exact(words, sig16, bits: int):
    """Exact layout -> regular layout: (words [n][4b] u32, meta [n] u32)."""
    words = np.ascontiguousarray(words, dtype=np.uint32).reshape(-1, 4 * bits)
    sig16 = np.ascontiguousarray(sig16, dtype=np.uint16).ravel()
    n = words.shape[0]
    out = np.empty_like(words)
    meta = np.empty(n, np.uint32)
    _load().oq_unfold_exact_batch(_p(words), _p(sig16), n, bits, _p(out), _p(meta))
    return out, meta

