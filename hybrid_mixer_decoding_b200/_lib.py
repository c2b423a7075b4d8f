"""ctypes binding of libhmd.so: the C ABI declared in include/hmd.h, same names, argument
marshalling only (shapes are read from the tensors, pointers and the current CUDA stream are
passed through). Every step of the mixers runs in the library's CUDA kernels; if the library is
missing, importing a function here raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os

import torch

FA, SWA, KDA, GDN = 0, 1, 2, 3
F32, BF16 = 0, 1
STATUS = {0: "HMD_OK", 1: "HMD_ERR_ARG", 2: "HMD_ERR_SHAPE", 3: "HMD_ERR_DTYPE",
          4: "HMD_ERR_OOM", 5: "HMD_ERR_CUDA", 6: "HMD_ERR_UNSUPPORTED",
          7: "HMD_ERR_DEVICE_CHECK"}
DEVERR_TIMEOUT, DEVERR_PAGE, DEVERR_SLOT, DEVERR_SEQLEN, DEVERR_GATE = 0x1, 0x2, 0x4, 0x8, 0x10

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhmd.so")
_lib = None

_c_int, _c_float, _vp, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class DeltaAct(ctypes.Structure):
    """hmd_delta_act_t: fused input activations of the delta-rule mixers."""
    _fields_ = [("A_log", _vp), ("dt_bias", _vp), ("l2_eps", _c_float)]


class DecodeIO(ctypes.Structure):
    """hmd_decode_io_t."""
    _fields_ = [("B", _c_int), ("H", _c_int), ("Hkv", _c_int), ("d", _c_int), ("dtype", _c_int),
                ("q", _vp), ("k", _vp), ("v", _vp), ("beta", _vp), ("log_gate_scalar", _vp),
                ("log_gate_channel", _vp), ("slots", _vp), ("page_table", _vp),
                ("max_pages", _c_int), ("seq_lens", _vp), ("max_seq_len", _c_int),
                ("window", _c_int), ("scale", _c_float), ("o", _vp)]


_SIGS = {
    "delta_rule_decode": (_c_int, [_c_int] * 6 + [_vp] * 6 + [_c_int, _vp, _vp, _c_float, _vp]),
    "hmd_group_sequences": (_c_int, [_c_int, _c_int, _vp, _c_int, _vp, _vp, _vp]),
    "batch_plan_create": (_c_int, [_c_int, _c_int, _vp, _c_int, _vp, _vp, ctypes.POINTER(_vp)]),
    "batch_plan_free": (_c_int, [_vp, _vp]),
    "batch_plan_group": (_c_int, [_vp, _c_int, _c_int, ctypes.POINTER(_c_int),
                                  ctypes.POINTER(ctypes.POINTER(ctypes.c_int32))]),
    "batch_plan_workspace_size": (_sz, [_vp] + [_c_int] * 6),
    "mixer_decode_step_batch": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "delta_rule_decode_act": (_c_int, [_c_int] * 6 + [_vp] * 7 + [_c_int, _vp, _vp, _vp,
                                                                 _c_float, _vp]),
    "delta_rule_prefill_chunked_act": (_c_int, [_c_int] * 7 + [_vp] * 7 + [_c_int, _vp, _vp,
                                                                          _c_int, _c_float, _vp]),
    "delta_rule_decode_chain": (_c_int, [_c_int] * 7 + [_vp] * 6 + [_vp, _c_int, _vp, _vp,
                                                                  _c_float, _vp]),
    "delta_rule_decode_to": (_c_int, [_c_int] * 6 + [_vp] * 6 + [_c_int, _vp, _vp, _vp, _c_float,
                                                                _vp]),
    "delta_rule_prefill_chunked": (_c_int, [_c_int] * 7 + [_vp] * 6 + [_c_int, _vp, _vp, _c_int,
                                                                      _c_float, _vp]),
    "delta_rule_prefill_workspace_size": (_sz, [_c_int] * 8),
    "delta_rule_prefill_chunked_ws": (_c_int, [_c_int] * 7 + [_vp] * 6 + [_c_int, _vp, _vp, _c_int,
                                                                         _c_float, _vp, _sz, _vp]),
    "attn_decode_workspace_size": (_sz, [_c_int] * 8),
    "attn_verify_workspace_size": (_sz, [_c_int] * 9),
    "attn_verify": (_c_int, [_c_int] * 9 + [_vp] * 5 + [_c_int, _vp, _c_int, _vp, _c_int, _vp,
                                             _vp, _sz, _vp]),
    "attn_decode": (_c_int, [_c_int] * 7 + [_vp] * 5 + [_c_int, _vp, _c_int, _vp, _c_int, _vp,
                                                      _vp, _sz, _vp]),
    "attn_prefill": (_c_int, [_c_int] * 8 + [_vp] * 5 + [_c_int, _vp, _c_int, _vp, _vp]),
    "attn_prefill_ext": (_c_int, [_c_int] * 8 + [_vp] * 4 + [_c_int, _vp, _vp, _c_int, _vp,
                                                             _c_int, _vp, _vp]),
    "attn_decode_static_ws": (_c_int, [_c_int] * 7 + [_vp] * 5 + [_c_int, _vp, _c_int, _vp,
                                                                _c_int, _vp, _vp]),
    "state_cache_alloc": (_c_int, [_c_int] * 5 + [_vp, ctypes.POINTER(_vp)]),
    "state_cache_free": (_c_int, [_vp, _vp]),
    "state_cache_save": (_c_int, [_vp, _c_int, _vp, _c_int, _vp, _vp]),
    "state_cache_layer": (_c_int, [_vp, _c_int, ctypes.POINTER(_vp)]),
    "state_cache_reset": (_c_int, [_vp, _c_int, _vp, _c_int, _vp, _vp]),
    "kv_cache_alloc": (_c_int, [_c_int, _vp] + [_c_int] * 5 + [_vp, ctypes.POINTER(_vp)]),
    "kv_cache_free": (_c_int, [_vp, _vp]),
    "kv_cache_layer": (_c_int, [_vp, _c_int, ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    "mixer_decode_step": (_c_int, [_vp, _c_int, _c_int, ctypes.POINTER(DecodeIO), _vp, _vp, _vp,
                                   _sz, _vp]),
    "hmd_status_string": (ctypes.c_char_p, [_c_int]),
    "hmd_last_error": (_c_int, []),
    "hmd_device_errors": (_c_int, [_vp, ctypes.POINTER(ctypes.c_uint32), _c_int]),
    "hmd_version": (ctypes.c_char_p, []),
    "hmd_test_arm_copy_skip": (_c_int, [_c_int, _c_int, ctypes.c_uint64]),
}


def lib() -> ctypes.CDLL:
    """Load libhmd.so (built in-tree by hybrid_mixer_decoding_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m hybrid_mixer_decoding_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class HmdError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {STATUS.get(status, status)}")
        self.status = status


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise HmdError(fn, st)


def _p(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported activation dtype {t.dtype}")


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def delta_rule_decode(kind, q, k, v, beta, log_gate, state, o, slots=None, scale=1.0,
                      stream=None) -> None:
    """One GDN/KDA decode token per sequence (see include/hmd.h). q,k [B,H,dk]; v,o [B,H,dv];
    beta [B,H]; log_gate [B,H] or [B,H,dk]; state [n_slots,H,dk,dv] fp32 (in place)."""
    _contig(q, k, v, beta, log_gate, state, o, slots)
    B, H, dk = q.shape
    dv = v.shape[-1]
    st = lib().delta_rule_decode(kind, B, H, dk, dv, _dtype_code(q), _p(q), _p(k), _p(v),
                                 _p(beta), _p(log_gate), _p(state), state.shape[0], _p(slots),
                                 _p(o), float(scale), _stream(stream))
    _check("delta_rule_decode", st)


def delta_rule_decode_to(kind, q, k, v, beta, log_gate, state, o, slots, dst_slots, scale=1.0,
                         stream=None) -> None:
    """delta_rule_decode reading slot slots[b] and writing the updated state to dst_slots[b]
    (see include/hmd.h); slots, dst_slots int32 [B] on the device."""
    _contig(q, k, v, beta, log_gate, state, o, slots, dst_slots)
    B, H, dk = q.shape
    dv = v.shape[-1]
    st = lib().delta_rule_decode_to(kind, B, H, dk, dv, _dtype_code(q), _p(q), _p(k), _p(v),
                                    _p(beta), _p(log_gate), _p(state), state.shape[0], _p(slots),
                                    _p(dst_slots), _p(o), float(scale), _stream(stream))
    _check("delta_rule_decode_to", st)


def delta_rule_decode_act(kind, q_raw, k_raw, v, beta_logit, gate_logit, A_log, dt_bias, state,
                          o, slots=None, dst_slots=None, scale=1.0, eps=1e-6,
                          stream=None) -> None:
    """delta_rule_decode_to on raw projections, the input activations fused in (see
    include/hmd.h): A_log [H]; dt_bias [H] (GDN) or [H, dk] (KDA), fp32 on the device."""
    _contig(q_raw, k_raw, v, beta_logit, gate_logit, A_log, dt_bias, state, o, slots, dst_slots)
    B, H, dk = q_raw.shape
    dv = v.shape[-1]
    act = DeltaAct(A_log.data_ptr(), dt_bias.data_ptr(), float(eps))
    st = lib().delta_rule_decode_act(kind, B, H, dk, dv, _dtype_code(q_raw), _p(q_raw), _p(k_raw),
                                     _p(v), _p(beta_logit), _p(gate_logit), ctypes.byref(act),
                                     _p(state), state.shape[0], _p(slots), _p(dst_slots), _p(o),
                                     float(scale), _stream(stream))
    _check("delta_rule_decode_act", st)


def delta_rule_prefill_chunked_act(kind, q_raw, k_raw, v, beta_logit, gate_logit, A_log, dt_bias,
                                   state, o, slots=None, chunk=64, scale=1.0, eps=1e-6,
                                   stream=None) -> None:
    """delta_rule_prefill_chunked on raw projections, the input activations fused into the
    chunk-parallel pass (bf16, dk = dv = 128, chunk 64; see include/hmd.h)."""
    _contig(q_raw, k_raw, v, beta_logit, gate_logit, A_log, dt_bias, state, o, slots)
    B, T, H, dk = q_raw.shape
    dv = v.shape[-1]
    act = DeltaAct(A_log.data_ptr(), dt_bias.data_ptr(), float(eps))
    st = lib().delta_rule_prefill_chunked_act(kind, B, T, H, dk, dv, _dtype_code(q_raw),
                                              _p(q_raw), _p(k_raw), _p(v), _p(beta_logit),
                                              _p(gate_logit), ctypes.byref(act), _p(state),
                                              state.shape[0], _p(slots), _p(o), int(chunk),
                                              float(scale), _stream(stream))
    _check("delta_rule_prefill_chunked_act", st)


def delta_rule_decode_chain(kind, q, k, v, beta, log_gate, state, o, chain, scale=1.0,
                            act=None, stream=None) -> None:
    """n_q decode tokens per sequence along a slot chain (see include/hmd.h): q, k
    [B,n_q,H,dk]; v, o [B,n_q,H,dv]; beta [B,n_q,H]; log_gate [B,n_q,H] or [B,n_q,H,dk];
    chain int32 [n_q+1, B]; act: None, or (A_log, dt_bias, eps) for raw projections."""
    _contig(q, k, v, beta, log_gate, state, o, chain)
    B, n_q, H, dk = q.shape
    dv = v.shape[-1]
    a = None
    if act is not None:
        a = ctypes.byref(DeltaAct(act[0].data_ptr(), act[1].data_ptr(), float(act[2])))
    st = lib().delta_rule_decode_chain(kind, n_q, B, H, dk, dv, _dtype_code(q), _p(q), _p(k),
                                       _p(v), _p(beta), _p(log_gate), a, _p(state),
                                       state.shape[0], _p(chain), _p(o), float(scale),
                                       _stream(stream))
    _check("delta_rule_decode_chain", st)


def delta_rule_prefill_chunked(kind, q, k, v, beta, log_gate, state, o, slots=None, chunk=64,
                               scale=1.0, stream=None) -> None:
    """Chunked GDN/KDA prefill (see include/hmd.h). q,k [B,T,H,dk]; v,o [B,T,H,dv];
    beta [B,T,H]; log_gate [B,T,H] or [B,T,H,dk]; state [n_slots,H,dk,dv] (in/out)."""
    _contig(q, k, v, beta, log_gate, state, o, slots)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    st = lib().delta_rule_prefill_chunked(kind, B, T, H, dk, dv, _dtype_code(q), _p(q), _p(k),
                                          _p(v), _p(beta), _p(log_gate), _p(state),
                                          state.shape[0], _p(slots), _p(o), int(chunk),
                                          float(scale), _stream(stream))
    _check("delta_rule_prefill_chunked", st)


def delta_rule_prefill_workspace_size(kind, B, T, H, dk, dv, dtype, chunk=64) -> int:
    return int(lib().delta_rule_prefill_workspace_size(kind, B, T, H, dk, dv, dtype, chunk))


def delta_rule_prefill_chunked_ws(kind, q, k, v, beta, log_gate, state, o, workspace, slots=None,
                                  chunk=64, scale=1.0, stream=None) -> None:
    """delta_rule_prefill_chunked with caller-owned scratch `workspace` (a device tensor; its
    byte size is passed, see include/hmd.h)."""
    _contig(q, k, v, beta, log_gate, state, o, slots, workspace)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().delta_rule_prefill_chunked_ws(kind, B, T, H, dk, dv, _dtype_code(q), _p(q), _p(k),
                                             _p(v), _p(beta), _p(log_gate), _p(state),
                                             state.shape[0], _p(slots), _p(o), int(chunk),
                                             float(scale), _p(workspace), ws_bytes,
                                             _stream(stream))
    _check("delta_rule_prefill_chunked_ws", st)


def attn_decode_workspace_size(kind, window, B, Hq, Hkv, d, page_tokens, max_seq_len) -> int:
    return int(lib().attn_decode_workspace_size(kind, window, B, Hq, Hkv, d, page_tokens,
                                                max_seq_len))


def attn_decode(kind, window, q, new_k, new_v, k_pool, v_pool, page_table, seq_lens,
                max_seq_len, o, workspace, stream=None) -> None:
    """FA/SWA decode over the paged bf16 cache, appending the new token (see include/hmd.h).
    q,o [B,Hq,d]; new_k,new_v [B,Hkv,d]; pools [n_pages,Hkv,page_tokens,d];
    page_table [B,max_pages] int32; seq_lens [B] int32; workspace uint8 tensor."""
    _contig(q, new_k, new_v, k_pool, v_pool, page_table, seq_lens, o, workspace)
    B, Hq, d = q.shape
    n_pages, Hkv, PT, _ = k_pool.shape
    st = lib().attn_decode(kind, int(window), B, Hq, Hkv, d, PT, _p(q), _p(new_k), _p(new_v),
                           _p(k_pool), _p(v_pool), n_pages, _p(page_table), page_table.shape[1],
                           _p(seq_lens), int(max_seq_len), _p(o), _p(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_decode", st)


def attn_verify_workspace_size(kind, window, n_q, B, Hq, Hkv, d, page_tokens, max_seq_len) -> int:
    return int(lib().attn_verify_workspace_size(kind, window, n_q, B, Hq, Hkv, d, page_tokens,
                                                max_seq_len))


def attn_verify(kind, window, ring_pages, q, new_k, new_v, k_pool, v_pool, page_table, seq_lens,
                max_seq_len, o, workspace, stream=None) -> None:
    """Verification pass of n_q new tokens per sequence (see include/hmd.h).
    q,o [B,n_q,Hq,d]; new_k,new_v [B,n_q,Hkv,d]; the rest as in attn_decode; ring_pages is the
    SWA ring's size in pages (ignored for FA)."""
    _contig(q, new_k, new_v, k_pool, v_pool, page_table, seq_lens, o, workspace)
    B, n_q, Hq, d = q.shape
    n_pages, Hkv, PT, _ = k_pool.shape
    st = lib().attn_verify(kind, int(window), int(ring_pages), n_q, B, Hq, Hkv, d, PT, _p(q),
                           _p(new_k), _p(new_v), _p(k_pool), _p(v_pool), n_pages, _p(page_table),
                           page_table.shape[1], _p(seq_lens), int(max_seq_len), _p(o),
                           _p(workspace), workspace.numel() * workspace.element_size(),
                           _stream(stream))
    _check("attn_verify", st)


def attn_decode_static_ws(kind, window, q, new_k, new_v, k_pool, v_pool, page_table, seq_lens,
                          max_seq_len, o, stream=None) -> None:
    """attn_decode with its workspace taken from the library's fixed device array instead of a
    caller buffer (for callers that cannot allocate device memory; see include/hmd.h)."""
    _contig(q, new_k, new_v, k_pool, v_pool, page_table, seq_lens, o)
    B, Hq, d = q.shape
    n_pages, Hkv, PT, _ = k_pool.shape
    st = lib().attn_decode_static_ws(kind, int(window), B, Hq, Hkv, d, PT, _p(q), _p(new_k),
                                     _p(new_v), _p(k_pool), _p(v_pool), n_pages, _p(page_table),
                                     page_table.shape[1], _p(seq_lens), int(max_seq_len), _p(o),
                                     _stream(stream))
    _check("attn_decode_static_ws", st)


def attn_prefill(kind, window, q, k, v, k_pool, v_pool, page_table, o, stream=None) -> None:
    """FA/SWA prefill of a prompt into an empty paged cache (see include/hmd.h).
    q,o [B,T,Hq,d]; k,v [B,T,Hkv,d] bf16; pools [n_pages,Hkv,page_tokens,d];
    page_table [B,max_pages] int32."""
    _contig(q, k, v, k_pool, v_pool, page_table, o)
    B, T, Hq, d = q.shape
    n_pages, Hkv, PT, _ = k_pool.shape
    st = lib().attn_prefill(kind, int(window), B, T, Hq, Hkv, d, PT, _p(q), _p(k), _p(v),
                            _p(k_pool), _p(v_pool), n_pages, _p(page_table), page_table.shape[1],
                            _p(o), _stream(stream))
    _check("attn_prefill", st)


def attn_prefill_ext(kind, window, q, k, v, prefix_lens, max_prefix, k_pool, v_pool, page_table,
                     o, stream=None) -> None:
    """attn_prefill after a cached prefix of prefix_lens[b] positions (device int32 [B],
    multiples of 64; see include/hmd.h)."""
    _contig(q, k, v, prefix_lens, k_pool, v_pool, page_table, o)
    B, T, Hq, d = q.shape
    n_pages, Hkv, PT, _ = k_pool.shape
    st = lib().attn_prefill_ext(kind, int(window), B, T, Hq, Hkv, d, PT, _p(q), _p(k), _p(v),
                                _p(prefix_lens), int(max_prefix), _p(k_pool), _p(v_pool), n_pages,
                                _p(page_table), page_table.shape[1], _p(o), _stream(stream))
    _check("attn_prefill_ext", st)


class StateCache:
    """state_cache_alloc / _layer / _reset / _free: n_layers x [slots,H,dk,dv] fp32."""

    def __init__(self, n_layers, slots, H, dk, dv, stream=None):
        h = _vp()
        _check("state_cache_alloc", lib().state_cache_alloc(n_layers, slots, H, dk, dv,
                                                            _stream(stream), ctypes.byref(h)))
        self.handle = h.value
        self.n_layers, self.slots, self.H, self.dk, self.dv = n_layers, slots, H, dk, dv

    def layer_ptr(self, layer) -> int:
        p = _vp()
        _check("state_cache_layer", lib().state_cache_layer(self.handle, layer, ctypes.byref(p)))
        return p.value

    def layer_view(self, layer) -> torch.Tensor:
        """A torch view of the layer's [slots,H,dk,dv] block (no copy)."""
        n = self.slots * self.H * self.dk * self.dv
        return _from_ptr(self.layer_ptr(layer), n, torch.float32).view(
            self.slots, self.H, self.dk, self.dv)

    def reset(self, layer, slot_ids, init=None, stream=None):
        ids = (ctypes.c_int32 * len(slot_ids))(*[int(s) for s in slot_ids])
        _check("state_cache_reset", lib().state_cache_reset(self.handle, layer, ids,
                                                            len(slot_ids), _p(init),
                                                            _stream(stream)))

    def save(self, layer, slot_ids, out, stream=None):
        """state_cache_save: copy the listed slots of one layer into out [n,H,dk,dv] fp32."""
        ids = (ctypes.c_int32 * len(slot_ids))(*[int(x) for x in slot_ids])
        _check("state_cache_save", lib().state_cache_save(self.handle, layer, ids, len(slot_ids),
                                                          _p(out), _stream(stream)))

    def free(self, stream=None):
        if self.handle:
            _check("state_cache_free", lib().state_cache_free(self.handle, _stream(stream)))
            self.handle = None


class KVCache:
    """kv_cache_alloc / _layer / _free: n_pools pairs of [n_pages,Hkv,page_tokens,d] bf16."""

    def __init__(self, layer_pool, n_pools, n_pages, Hkv, d, page_tokens=64, stream=None):
        lp = (ctypes.c_int32 * len(layer_pool))(*[int(x) for x in layer_pool])
        h = _vp()
        _check("kv_cache_alloc", lib().kv_cache_alloc(len(layer_pool), lp, n_pools, n_pages, Hkv,
                                                      d, page_tokens, _stream(stream),
                                                      ctypes.byref(h)))
        self.handle = h.value
        self.n_pages, self.Hkv, self.d, self.page_tokens = n_pages, Hkv, d, page_tokens

    def layer_pools(self, layer):
        kp, vp = _vp(), _vp()
        _check("kv_cache_layer", lib().kv_cache_layer(self.handle, layer, ctypes.byref(kp),
                                                      ctypes.byref(vp)))
        n = self.n_pages * self.Hkv * self.page_tokens * self.d
        shape = (self.n_pages, self.Hkv, self.page_tokens, self.d)
        return (_from_ptr(kp.value, n, torch.bfloat16).view(shape),
                _from_ptr(vp.value, n, torch.bfloat16).view(shape))

    def free(self, stream=None):
        if self.handle:
            _check("kv_cache_free", lib().kv_cache_free(self.handle, _stream(stream)))
            self.handle = None


def _from_ptr(ptr: int, n: int, dtype) -> torch.Tensor:
    """Wrap library-owned device memory as a torch tensor (no copy, no ownership)."""
    class _CAI:
        __cuda_array_interface__ = {
            "shape": (n,), "typestr": {torch.float32: "<f4", torch.bfloat16: "<i2"}[dtype],
            "data": (ptr, False), "version": 3, "strides": None}
    t = torch.as_tensor(_CAI(), device="cuda")
    return t.view(dtype) if dtype == torch.bfloat16 else t


def mixer_decode_step(placement, layer, io: DecodeIO, state_cache=None, kv_cache=None,
                      workspace=None, stream=None) -> None:
    """Run layer `layer`'s mixer as chosen by placement (host int8 array) on its caches."""
    pl = placement if isinstance(placement, ctypes.Array) else \
        (ctypes.c_int8 * len(placement))(*[int(x) for x in placement])
    ws = _p(workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().mixer_decode_step(pl, len(pl), layer, ctypes.byref(io),
                                 state_cache.handle if state_cache else None,
                                 kv_cache.handle if kv_cache else None, ws, ws_bytes,
                                 _stream(stream))
    _check("mixer_decode_step", st)


def group_sequences(placements, seq_placement):
    """hmd_group_sequences (host only): placements int8 [n_placements][n_layers], seq_placement
    int32 [B] -> (rows int32 [n_layers][B], offsets int32 [n_layers][5])."""
    import numpy as np
    pl = np.ascontiguousarray(placements, dtype=np.int8)
    sp = np.ascontiguousarray(seq_placement, dtype=np.int32)
    n_p, n_l = pl.shape
    B = sp.shape[0]
    rows = np.zeros((n_l, B), np.int32)
    offs = np.zeros((n_l, 5), np.int32)
    _check("hmd_group_sequences", lib().hmd_group_sequences(
        n_l, n_p, pl.ctypes.data, B, sp.ctypes.data, rows.ctypes.data, offs.ctypes.data))
    return rows, offs


class BatchPlan:
    """batch_plan_create / _group / _workspace_size / _free: the per-layer grouping of a
    mixed batch's sequences by mixer kind, with the rows on the device."""

    def __init__(self, placements, seq_placement, stream=None):
        import numpy as np
        pl = np.ascontiguousarray(placements, dtype=np.int8)
        sp = np.ascontiguousarray(seq_placement, dtype=np.int32)
        self.n_layers, self.B = pl.shape[1], sp.shape[0]
        h = _vp()
        _check("batch_plan_create", lib().batch_plan_create(self.n_layers, pl.shape[0],
                                                            pl.ctypes.data, self.B,
                                                            sp.ctypes.data, _stream(stream),
                                                            ctypes.byref(h)))
        self.handle = h.value

    def group(self, layer, kind):
        import numpy as np
        n = _c_int()
        ptr = ctypes.POINTER(ctypes.c_int32)()
        _check("batch_plan_group", lib().batch_plan_group(self.handle, layer, kind,
                                                          ctypes.byref(n), ctypes.byref(ptr)))
        return np.ctypeslib.as_array(ptr, shape=(n.value,)).copy() if n.value else \
            np.zeros(0, np.int32)

    def workspace_size(self, window, Hq, Hkv, d, page_tokens, max_seq_len) -> int:
        return int(lib().batch_plan_workspace_size(self.handle, window, Hq, Hkv, d, page_tokens,
                                                   max_seq_len))

    def free(self, stream=None):
        if self.handle:
            _check("batch_plan_free", lib().batch_plan_free(self.handle, _stream(stream)))
            self.handle = None


def mixer_decode_step_batch(plan: BatchPlan, layer, ios, state_cache=None, kv_cache=None,
                            workspace=None, stream=None) -> None:
    """One decode token for layer `layer` of a mixed batch: ios maps each kind present at the
    layer to its DecodeIO (full-batch tensors)."""
    arr = (ctypes.POINTER(DecodeIO) * 4)()
    for kind, io in ios.items():
        arr[kind] = ctypes.pointer(io)
    ws = _p(workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().mixer_decode_step_batch(plan.handle, layer, ctypes.cast(arr, _vp),
                                       state_cache.handle if state_cache else None,
                                       kv_cache.handle if kv_cache else None, ws, ws_bytes,
                                       _stream(stream))
    _check("mixer_decode_step_batch", st)


def hmd_device_errors(clear=True, stream=None) -> int:
    bits = ctypes.c_uint32()
    _check("hmd_device_errors", lib().hmd_device_errors(_stream(stream), ctypes.byref(bits),
                                                        1 if clear else 0))
    return int(bits.value)


def hmd_status_string(status: int) -> str:
    return lib().hmd_status_string(status).decode()


def hmd_last_error() -> int:
    return int(lib().hmd_last_error())


def hmd_version() -> str:
    return lib().hmd_version().decode()


TEST_DELTA_DECODE, TEST_ATTN_SPLIT = 0, 1


def hmd_test_arm_copy_skip(kernel: int, cta: int, wait_ns: int) -> None:
    """Arm a one-shot missing copy in CTA `cta` of this thread's next launch of `kernel`
    (TEST_DELTA_DECODE or TEST_ATTN_SPLIT), with every bounded wait of that launch limited to
    wait_ns: the failure-detection tests' way to make a wait run out without an invalid access."""
    _check("hmd_test_arm_copy_skip", lib().hmd_test_arm_copy_skip(kernel, cta, wait_ns))
