"""Thin ctypes binding of liblkv (include/lkv.h).

Functions carry the C names and argument order.  Tensor arguments may be
torch tensors (their data_ptr() is passed) or raw integer addresses; the
stream defaults to torch's current CUDA stream.  A nonzero status raises
LkvError.  This module only marshals arguments: every step of the path runs
in the CUDA kernels of liblkv.so, and there is no fallback -- if the library
is missing, every call raises.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblkv.so")

LKV_OK = 0
LKV_ERR_INVALID_ARG = 1
LKV_ERR_UNSUPPORTED = 2
LKV_ERR_WORKSPACE = 3
LKV_ERR_CUDA = 4
LKV_ERR_TIMEOUT = 5


class LkvError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {lkv_status_string(status)} ({status})")


class lkv_qspec(ctypes.Structure):
    _fields_ = [("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32), ("group", ctypes.c_int32)]


class lkv_segment(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("k_sz", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_sz", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t

# name -> (restype, argtypes); this table mirrors include/lkv.h.
SIGNATURES = {
    "lkv_status_string": (ctypes.c_char_p, [_I]),
    "lkv_version": (_I, []),
    "lkv_row_bytes": (_Z, [_I, _I]),
    "lkv_sz_row_bytes": (_Z, [_I, _I]),
    "lkv_quantize_kv": (_I, [lkv_qspec, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "lkv_append_kv": (_I, [lkv_qspec, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "lkv_quantize_kv_paged": (_I, [lkv_qspec, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "lkv_append_kv_paged": (_I, [lkv_qspec, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "lkv_decode_attention_paged": (_I, [lkv_qspec, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _F,
                                        _F, _P, _P, _P, _P, _Z, _P]),
    "lkv_decode_workspace_bytes": (_Z, [lkv_qspec, _I, _I, _I, _I, _I]),
    "lkv_decode_attention": (_I, [lkv_qspec, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _F, _F,
                                  _P, _P, _P, _P, _Z, _P]),
    "lkv_decode_attention_mass": (_I, [lkv_qspec, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _F, _F,
                                       _P, _P, _P, _P, _P, _Z, _P]),
    "lkv_decode_attention_static": (_I, [lkv_qspec, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _F,
                                         _F, _P, _P, _P, _P, _P]),
    "lkv_workspace_reset": (_I, [_P, _Z, _P]),
    "lkv_workspace_status": (_I, [_P, _P, _P]),
    "lkv_tier_classify": (_I, [_I, _I, _I, _P, _P, _F, _F, _P, _P, _P, _P, _P]),
    "lkv_tier_repack": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, lkv_segment, lkv_segment, _P]),
    "lkv_tiered_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I]),
    "lkv_tiered_attention": (_I, [_I, _I, _I, _I, _I, _I, _P, _P, lkv_segment, lkv_segment, _F, _F,
                                  _P, _P, _P, _Z, _P]),
    "lkv_tiered_decode": (_I, [_I, _I, _I, _I, _I, _I, _P, _P, _F, _F, _P, _P, _P, _P, _P, _P, _P,
                               lkv_segment, lkv_segment, _F, _F, _P, _P, _P, _Z, _P]),
}

_lib = None


def lib():
    """The loaded liblkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m quantized_kv_cache_lkv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc, what):
    if rc != LKV_OK:
        raise LkvError(rc, what)


def _spec(spec):
    if isinstance(spec, lkv_qspec):
        return spec
    kb, vb, g = spec
    return lkv_qspec(kb, vb, g)


def _seg(seg):
    if isinstance(seg, lkv_segment):
        return seg
    return lkv_segment(_ptr(seg["k_codes"]), _ptr(seg["k_sz"]), _ptr(seg["v_codes"]), _ptr(seg["v_sz"]))


def lkv_status_string(status):
    return lib().lkv_status_string(status).decode()


def lkv_version():
    return lib().lkv_version()


def lkv_row_bytes(bits, D):
    return lib().lkv_row_bytes(bits, D)


def lkv_sz_row_bytes(D, group):
    return lib().lkv_sz_row_bytes(D, group)


def lkv_quantize_kv(spec, B, Hkv, T_cap, D, seq_lens, k, v, k_codes, k_sz, v_codes, v_sz, stream=None):
    _check(lib().lkv_quantize_kv(_spec(spec), B, Hkv, T_cap, D, _ptr(seq_lens), _ptr(k), _ptr(v),
                                 _ptr(k_codes), _ptr(k_sz), _ptr(v_codes), _ptr(v_sz),
                                 _stream(stream)), "lkv_quantize_kv")


def lkv_append_kv(spec, B, Hkv, T_cap, D, pos, k_new, v_new, k_codes, k_sz, v_codes, v_sz, stream=None):
    _check(lib().lkv_append_kv(_spec(spec), B, Hkv, T_cap, D, _ptr(pos), _ptr(k_new), _ptr(v_new),
                               _ptr(k_codes), _ptr(k_sz), _ptr(v_codes), _ptr(v_sz), _stream(stream)),
           "lkv_append_kv")


LKV_PAGE_TOKENS = 256


def lkv_quantize_kv_paged(spec, B, Hkv, pages_per_seq, num_pages, D, seq_lens, k, v, block_table, k_pool,
                          k_sz_pool, v_pool, v_sz_pool, stream=None):
    _check(lib().lkv_quantize_kv_paged(_spec(spec), B, Hkv, pages_per_seq, num_pages, D, _ptr(seq_lens),
                                       _ptr(k), _ptr(v), _ptr(block_table), _ptr(k_pool), _ptr(k_sz_pool),
                                       _ptr(v_pool), _ptr(v_sz_pool), _stream(stream)), "lkv_quantize_kv_paged")


def lkv_append_kv_paged(spec, B, Hkv, pages_per_seq, num_pages, D, pos, k_new, v_new, block_table, k_pool,
                        k_sz_pool, v_pool, v_sz_pool, stream=None):
    _check(lib().lkv_append_kv_paged(_spec(spec), B, Hkv, pages_per_seq, num_pages, D, _ptr(pos), _ptr(k_new),
                                     _ptr(v_new), _ptr(block_table), _ptr(k_pool), _ptr(k_sz_pool),
                                     _ptr(v_pool), _ptr(v_sz_pool), _stream(stream)), "lkv_append_kv_paged")


def lkv_decode_attention_paged(spec, B, Hq, Hkv, pages_per_seq, num_pages, D, seq_lens, q, block_table, k_pool,
                               k_sz_pool, v_pool, v_sz_pool, softmax_scale, tau, out, skip_mask, skip_counts,
                               workspace, ws_bytes, stream=None):
    _check(lib().lkv_decode_attention_paged(_spec(spec), B, Hq, Hkv, pages_per_seq, num_pages, D,
                                            _ptr(seq_lens), _ptr(q), _ptr(block_table), _ptr(k_pool),
                                            _ptr(k_sz_pool), _ptr(v_pool), _ptr(v_sz_pool), float(softmax_scale),
                                            float(tau), _ptr(out), _ptr(skip_mask), _ptr(skip_counts),
                                            _ptr(workspace), int(ws_bytes), _stream(stream)),
           "lkv_decode_attention_paged")


def lkv_decode_workspace_bytes(spec, B, Hq, Hkv, T_cap, D):
    return lib().lkv_decode_workspace_bytes(_spec(spec), B, Hq, Hkv, T_cap, D)


def lkv_decode_attention(spec, B, Hq, Hkv, T_cap, D, seq_lens, q, k_codes, k_sz, v_codes, v_sz,
                         softmax_scale, tau, out, skip_mask, skip_counts, workspace, ws_bytes,
                         stream=None):
    _check(lib().lkv_decode_attention(_spec(spec), B, Hq, Hkv, T_cap, D, _ptr(seq_lens), _ptr(q),
                                      _ptr(k_codes), _ptr(k_sz), _ptr(v_codes), _ptr(v_sz),
                                      float(softmax_scale), float(tau), _ptr(out), _ptr(skip_mask),
                                      _ptr(skip_counts), _ptr(workspace), int(ws_bytes),
                                      _stream(stream)), "lkv_decode_attention")


def lkv_decode_attention_mass(spec, B, Hq, Hkv, T_cap, D, seq_lens, q, k_codes, k_sz, v_codes, v_sz,
                              softmax_scale, tau, out, skip_mask, skip_counts, mass, workspace, ws_bytes,
                              stream=None):
    _check(lib().lkv_decode_attention_mass(_spec(spec), B, Hq, Hkv, T_cap, D, _ptr(seq_lens), _ptr(q),
                                           _ptr(k_codes), _ptr(k_sz), _ptr(v_codes), _ptr(v_sz),
                                           float(softmax_scale), float(tau), _ptr(out), _ptr(skip_mask),
                                           _ptr(skip_counts), _ptr(mass), _ptr(workspace), int(ws_bytes),
                                           _stream(stream)), "lkv_decode_attention_mass")


LKV_STATIC_WORKSPACE_BYTES = 32 << 20


def lkv_decode_attention_static(spec, B, Hq, Hkv, T_cap, D, seq_lens, q, k_codes, k_sz, v_codes, v_sz,
                                softmax_scale, tau, out, skip_mask, skip_counts, status, stream=None):
    _check(lib().lkv_decode_attention_static(_spec(spec), B, Hq, Hkv, T_cap, D, _ptr(seq_lens), _ptr(q),
                                             _ptr(k_codes), _ptr(k_sz), _ptr(v_codes), _ptr(v_sz),
                                             float(softmax_scale), float(tau), _ptr(out),
                                             _ptr(skip_mask), _ptr(skip_counts), _ptr(status),
                                             _stream(stream)), "lkv_decode_attention_static")


def lkv_workspace_reset(workspace, ws_bytes, stream=None):
    _check(lib().lkv_workspace_reset(_ptr(workspace), int(ws_bytes), _stream(stream)),
           "lkv_workspace_reset")


def lkv_workspace_status(workspace, stream=None):
    """Returns the device status word (an lkv status code); synchronizes the stream."""
    st = ctypes.c_int32(0)
    _check(lib().lkv_workspace_status(_ptr(workspace), _stream(stream), ctypes.addressof(st)),
           "lkv_workspace_status")
    return st.value


def lkv_tier_classify(B, Hkv, T_cap, seq_lens, mass, tau_low, tau_high, tier, counts, pos_a, pos_b,
                      stream=None):
    _check(lib().lkv_tier_classify(B, Hkv, T_cap, _ptr(seq_lens), _ptr(mass), float(tau_low),
                                   float(tau_high), _ptr(tier), _ptr(counts), _ptr(pos_a), _ptr(pos_b),
                                   _stream(stream)), "lkv_tier_classify")


def lkv_tier_repack(B, Hkv, T_cap, D, group, k, v, counts, pos_a, pos_b, seg_a, seg_b, stream=None):
    _check(lib().lkv_tier_repack(B, Hkv, T_cap, D, group, _ptr(k), _ptr(v), _ptr(counts), _ptr(pos_a),
                                 _ptr(pos_b), _seg(seg_a), _seg(seg_b), _stream(stream)),
           "lkv_tier_repack")


def lkv_tiered_workspace_bytes(B, Hq, Hkv, T_cap, D, group):
    return lib().lkv_tiered_workspace_bytes(B, Hq, Hkv, T_cap, D, group)


def lkv_tiered_attention(B, Hq, Hkv, T_cap, D, group, counts, q, seg_a, seg_b, softmax_scale, tau, out,
                         skip_counts, workspace, ws_bytes, stream=None):
    _check(lib().lkv_tiered_attention(B, Hq, Hkv, T_cap, D, group, _ptr(counts), _ptr(q), _seg(seg_a),
                                      _seg(seg_b), float(softmax_scale), float(tau), _ptr(out),
                                      _ptr(skip_counts), _ptr(workspace), int(ws_bytes),
                                      _stream(stream)), "lkv_tiered_attention")


def lkv_tiered_decode(B, Hq, Hkv, T_cap, D, group, seq_lens, mass, tau_low, tau_high, k, v, q, tier,
                      counts, pos_a, pos_b, seg_a, seg_b, softmax_scale, tau, out, skip_counts,
                      workspace, ws_bytes, stream=None):
    _check(lib().lkv_tiered_decode(B, Hq, Hkv, T_cap, D, group, _ptr(seq_lens), _ptr(mass),
                                   float(tau_low), float(tau_high), _ptr(k), _ptr(v), _ptr(q),
                                   _ptr(tier), _ptr(counts), _ptr(pos_a), _ptr(pos_b), _seg(seg_a),
                                   _seg(seg_b), float(softmax_scale), float(tau), _ptr(out),
                                   _ptr(skip_counts), _ptr(workspace), int(ws_bytes),
                                   _stream(stream)), "lkv_tiered_decode")
