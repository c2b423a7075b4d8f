"""ctypes wrapper around the fp64 C oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg are
the only callers. Nothing here is used by the library's product path, and this module imports
nothing from the library package.

Inputs are upcast to float64 exactly (fp32 and bf16 values are representable in fp64); the C
code does every operation of the method in fp64. See oracle.c for the definitions followed and
the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

FA, SWA, KDA, GDN = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, fp64, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIB points the pins at another build of oracle.c (the mutation test uses it
        # to check that deliberately broken copies fail the pins).
        path = os.environ.get("ORACLE_LIB")
        if not path:
            path = build()
        lib = ctypes.CDLL(path)
        D = ctypes.POINTER(ctypes.c_double)
        I32 = ctypes.POINTER(ctypes.c_int32)
        U16 = ctypes.POINTER(ctypes.c_uint16)
        c_int, c_double = ctypes.c_int, ctypes.c_double
        lib.oracle_delta_recurrent.argtypes = [c_int] * 6 + [D] * 5 + [c_double, D, D, c_int]
        lib.oracle_delta_chunked.argtypes = [c_int] * 7 + [D] * 5 + [c_double, D, D, c_int]
        lib.oracle_kv_slot.argtypes = [c_int, c_int, c_int, I32, c_int, c_int, I32, I32]
        lib.oracle_attn_decode.argtypes = ([c_int] * 8 + [D, D, D, U16, U16, I32, c_int, I32, D,
                                                          c_int])
        lib.oracle_attn_prefill.argtypes = [c_int] * 7 + [D, D, D, D, c_int]
        lib.oracle_kv_slot_ring.argtypes = [c_int, c_int, c_int, I32, c_int, c_int, I32, I32]
        lib.oracle_attn_verify.argtypes = ([c_int] * 10 + [D, D, D, U16, U16, I32, c_int, I32, D,
                                                           c_int])
        lib.oracle_delta_activations.argtypes = [c_int] * 4 + [c_double] + [D] * 10
        lib.oracle_max_threads.argtypes = []
        for f in ("oracle_delta_recurrent", "oracle_delta_chunked", "oracle_kv_slot",
                  "oracle_attn_decode", "oracle_attn_prefill", "oracle_kv_slot_ring",
                  "oracle_attn_verify", "oracle_delta_activations", "oracle_max_threads"):
            getattr(lib, f).restype = c_int
        _lib = lib
    return _lib


def _d(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(
        np.float32).astype(np.float64)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def delta_recurrent(kind, q, k, v, beta, log_gate, state0, scale=1.0, n_threads=0):
    """Token-by-token GDN/KDA. q,k [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H];
    log_gate [B,T,H] (GDN) or [B,T,H,dk] (KDA); state0 [B,H,dk,dv].
    Returns (o [B,T,H,dv], final state [B,H,dk,dv]) in float64."""
    q, k, v, beta, lg = _d(q), _d(k), _d(v), _d(beta), _d(log_gate)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    st = _d(state0).copy()
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    rc = _load().oracle_delta_recurrent(kind, B, T, H, dk, dv, _p(q, ctypes.c_double),
                                        _p(k, ctypes.c_double), _p(v, ctypes.c_double),
                                        _p(beta, ctypes.c_double), _p(lg, ctypes.c_double),
                                        float(scale), _p(st, ctypes.c_double),
                                        _p(o, ctypes.c_double), int(n_threads))
    if rc:
        raise ValueError("oracle_delta_recurrent failed")
    return o, st


def delta_chunked(kind, q, k, v, beta, log_gate, state0, chunk, scale=1.0, n_threads=0):
    """Chunked (UT-transform) GDN/KDA; same layouts and result as delta_recurrent."""
    q, k, v, beta, lg = _d(q), _d(k), _d(v), _d(beta), _d(log_gate)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    st = _d(state0).copy()
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    rc = _load().oracle_delta_chunked(kind, B, T, H, dk, dv, int(chunk), _p(q, ctypes.c_double),
                                      _p(k, ctypes.c_double), _p(v, ctypes.c_double),
                                      _p(beta, ctypes.c_double), _p(lg, ctypes.c_double),
                                      float(scale), _p(st, ctypes.c_double),
                                      _p(o, ctypes.c_double), int(n_threads))
    if rc:
        raise ValueError("oracle_delta_chunked failed")
    return o, st


def kv_slot(kind, window, page_tokens, page_row, pos):
    """(physical page, offset) of logical position pos for one sequence's page-table row."""
    row = np.ascontiguousarray(page_row, dtype=np.int32)
    pg, off = ctypes.c_int32(), ctypes.c_int32()
    rc = _load().oracle_kv_slot(kind, int(window), int(page_tokens),
                                _p(row, ctypes.c_int32), int(row.shape[0]), int(pos),
                                ctypes.byref(pg), ctypes.byref(off))
    if rc:
        raise ValueError("oracle_kv_slot: bad arguments")
    return int(pg.value), int(off.value)


def attn_decode(kind, window, q_bits, new_k_bits, new_v_bits, k_pool, v_pool, page_table,
                seq_lens, n_threads=0):
    """FA/SWA decode over a paged bf16 cache (see oracle.c). q_bits [B,Hq,d] and
    new_k/new_v_bits [B,Hkv,d] are bf16 bit patterns; k_pool/v_pool uint16 [P,Hkv,PT,d].
    Returns o [B,Hq,d] float64."""
    q = bf16_bits_to_f64(q_bits)
    nk = bf16_bits_to_f64(new_k_bits)
    nv = bf16_bits_to_f64(new_v_bits)
    kp = np.ascontiguousarray(k_pool, dtype=np.uint16)
    vp = np.ascontiguousarray(v_pool, dtype=np.uint16)
    pt_ = np.ascontiguousarray(page_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, d = q.shape
    P, Hkv, PT, _ = kp.shape
    o = np.zeros((B, Hq, d), dtype=np.float64)
    rc = _load().oracle_attn_decode(kind, int(window), B, Hq, Hkv, d, PT, P,
                                    _p(q, ctypes.c_double), _p(nk, ctypes.c_double),
                                    _p(nv, ctypes.c_double), _p(kp, ctypes.c_uint16),
                                    _p(vp, ctypes.c_uint16), _p(pt_, ctypes.c_int32),
                                    int(pt_.shape[1]), _p(sl, ctypes.c_int32),
                                    _p(o, ctypes.c_double), int(n_threads))
    if rc:
        raise ValueError("oracle_attn_decode failed (bad arguments or page id)")
    return o


def attn_prefill(kind, window, q, k, v, n_threads=0):
    """FA/SWA prefill from an empty cache (see oracle.c): q [B,T,Hq,d], k, v [B,T,Hkv,d]
    (float64; pass the exact values the GPU receives). Returns o [B,T,Hq,d] float64."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    o = np.zeros((B, T, Hq, d), dtype=np.float64)
    rc = _load().oracle_attn_prefill(kind, int(window), B, T, Hq, Hkv, d, _p(q, ctypes.c_double),
                                     _p(k, ctypes.c_double), _p(v, ctypes.c_double),
                                     _p(o, ctypes.c_double), int(n_threads))
    if rc:
        raise ValueError("oracle_attn_prefill: bad arguments")
    return o


def kv_slot_ring(kind, ring_pages, page_tokens, page_row, pos):
    """(physical page, offset) of logical position pos with an SWA ring of ring_pages pages."""
    row = np.ascontiguousarray(page_row, dtype=np.int32)
    pg, off = ctypes.c_int32(), ctypes.c_int32()
    rc = _load().oracle_kv_slot_ring(kind, int(ring_pages), int(page_tokens),
                                     _p(row, ctypes.c_int32), int(row.shape[0]), int(pos),
                                     ctypes.byref(pg), ctypes.byref(off))
    if rc:
        raise ValueError("oracle_kv_slot_ring: bad arguments")
    return int(pg.value), int(off.value)


def attn_verify(kind, window, ring_pages, q_bits, new_k_bits, new_v_bits, k_pool, v_pool,
                page_table, seq_lens, n_threads=0):
    """Verification of n_q tokens per sequence (see oracle.c): q_bits [B,n_q,Hq,d] and
    new_k/new_v_bits [B,n_q,Hkv,d] bf16 bit patterns; pools uint16 [P,Hkv,PT,d] holding
    positions 0..L-n_q-1. Returns o [B,n_q,Hq,d] float64."""
    q = bf16_bits_to_f64(q_bits)
    nk = bf16_bits_to_f64(new_k_bits)
    nv = bf16_bits_to_f64(new_v_bits)
    kp = np.ascontiguousarray(k_pool, dtype=np.uint16)
    vp = np.ascontiguousarray(v_pool, dtype=np.uint16)
    pt_ = np.ascontiguousarray(page_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, n_q, Hq, d = q.shape
    P, Hkv, PT, _ = kp.shape
    o = np.zeros((B, n_q, Hq, d), dtype=np.float64)
    rc = _load().oracle_attn_verify(kind, int(window), int(ring_pages), n_q, B, Hq, Hkv, d, PT, P,
                                    _p(q, ctypes.c_double), _p(nk, ctypes.c_double),
                                    _p(nv, ctypes.c_double), _p(kp, ctypes.c_uint16),
                                    _p(vp, ctypes.c_uint16), _p(pt_, ctypes.c_int32),
                                    int(pt_.shape[1]), _p(sl, ctypes.c_int32),
                                    _p(o, ctypes.c_double), int(n_threads))
    if rc:
        raise ValueError("oracle_attn_verify failed (bad arguments or page id)")
    return o


def delta_activations(kind, q_raw, k_raw, beta_logit, gate_logit, A_log, dt_bias, eps=1e-6):
    """Input activations of GDN/KDA from raw projections (see oracle.c): q_raw, k_raw
    [..., H, dk]; beta_logit [..., H]; gate_logit [..., H] (GDN) or [..., H, dk] (KDA);
    A_log [H]; dt_bias [H] or [H, dk]. Returns (q, k, beta, log_gate) in float64, same shapes."""
    qr, kr = _d(q_raw), _d(k_raw)
    bl, gl, al, db = _d(beta_logit), _d(gate_logit), _d(A_log), _d(dt_bias)
    H, dk = qr.shape[-2], qr.shape[-1]
    N = qr.size // (H * dk)
    q, k = np.zeros_like(qr), np.zeros_like(kr)
    beta, lg = np.zeros_like(bl), np.zeros_like(gl)
    rc = _load().oracle_delta_activations(kind, N, H, dk, float(eps), _p(qr, ctypes.c_double),
                                          _p(kr, ctypes.c_double), _p(bl, ctypes.c_double),
                                          _p(gl, ctypes.c_double), _p(al, ctypes.c_double),
                                          _p(db, ctypes.c_double), _p(q, ctypes.c_double),
                                          _p(k, ctypes.c_double), _p(beta, ctypes.c_double),
                                          _p(lg, ctypes.c_double))
    if rc:
        raise ValueError("oracle_delta_activations: bad arguments")
    return q, k, beta, lg


# Every rel_err call is logged here with the elementwise figure beside the normwise one; the
# test session prints the worst of each per test (tests/conftest.py).
PARITY_LOG: list = []
PARITY_LABEL = [""]  # the running test's id, set by the test session


def elementwise_p99(x, ref) -> float:
    """99th percentile over the elements of |x - ref| / max(|ref|, 1e-6 max|ref|): the
    elementwise relative error, with an absolute floor so that entries near zero do not make it
    undefined. Logged beside the normwise measure; the tolerances apply to the normwise one."""
    x = np.asarray(x, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    if ref.size == 0:
        return 0.0
    floor = 1e-6 * float(np.max(np.abs(ref)))
    den = np.maximum(np.abs(ref), floor)
    with np.errstate(divide="ignore", invalid="ignore"):
        e = np.abs(x - ref) / den
    e = np.where(den > 0, e, np.abs(x - ref))
    return float(np.percentile(e, 99))


def rel_err(x, ref) -> float:
    """Normwise relative error max|x - ref| / max|ref| (the parity measure). The elementwise
    p99 (elementwise_p99) is logged beside it in PARITY_LOG."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(x - ref))) if ref.size else 0.0
    r = num / den if den > 0 else num
    PARITY_LOG.append({"test": PARITY_LABEL[0], "shape": list(ref.shape), "normwise": r,
                       "p99_elementwise": elementwise_p99(x, ref)})
    return r
