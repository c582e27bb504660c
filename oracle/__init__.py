"""CPU oracle for the quantized-KV decode path (TEST INFRASTRUCTURE ONLY).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline may import this package.  The product path (the CUDA library and its
Python binding) never does, and shares no code with it.

The arithmetic lives in ``lkv_oracle.c`` (plain loops: an fp32 quantizer that
rounds every operation on its own, fp64 attention).  This module only moves
numpy arrays across ctypes.  bf16 tensors are passed as their raw uint16 bits.

Sources: "Super KV Compression: 突破LLM推理内存瓶颈的三层压缩架构解析"
(§第一层 asymmetric K6V4 quantization, §第二层 attention tiers, §第三层
sparse-V skip) and "TurboQuant：将LLM KV缓存压缩5-7倍的突破性技术"
(§TurboQuant的核心创新, asymmetric group-wise quantization).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.lkv_oracle_row_bytes.restype = ctypes.c_longlong
        L.lkv_oracle_row_bytes.argtypes = [_I, _I]
        L.lkv_oracle_quantize_group.restype = None
        L.lkv_oracle_quantize_group.argtypes = [_P, _I, _I, _P, _P, _P]
        L.lkv_oracle_dequant.restype = _F
        L.lkv_oracle_dequant.argtypes = [ctypes.c_uint32, _F, _F]
        L.lkv_oracle_pack_row.restype = None
        L.lkv_oracle_pack_row.argtypes = [_P, _I, _I, _P]
        L.lkv_oracle_unpack_row.restype = None
        L.lkv_oracle_unpack_row.argtypes = [_P, _I, _I, _P]
        L.lkv_oracle_dequant_rows.restype = _I
        L.lkv_oracle_dequant_rows.argtypes = [_P, _P, ctypes.c_longlong, _I, _I, _I, _P]
        L.lkv_oracle_quantize_kv.restype = _I
        L.lkv_oracle_quantize_kv.argtypes = [_I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]
        L.lkv_oracle_decode_attention.restype = _I
        L.lkv_oracle_decode_attention.argtypes = [_I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                                  _P, _P, _F, _F, _P, _P, _P, _P]
        L.lkv_oracle_tier_classify.restype = _I
        L.lkv_oracle_tier_classify.argtypes = [_I, _I, _I, _P, _P, _F, _F, _P, _P, _P, _P]
        L.lkv_oracle_tier_repack.restype = _I
        L.lkv_oracle_tier_repack.argtypes = [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                                             _P, _P, _P, _P, _P, _P, _P, _P]
        L.lkv_oracle_tiered_attention.restype = _I
        L.lkv_oracle_tiered_attention.argtypes = [_I, _I, _I, _I, _I, _I, _P, _P,
                                                  _P, _P, _P, _P, _P, _P, _P, _P,
                                                  _F, _F, _P, _P, _P]
        L.lkv_oracle_attention_bf16.restype = _I
        L.lkv_oracle_attention_bf16.argtypes = [_I, _I, _I, _I, _I, _P, _P, _P, _P, _F, _P]
        L.lkv_oracle_set_threads.restype = None
        L.lkv_oracle_set_threads.argtypes = [_I]
        L.lkv_oracle_get_threads.restype = _I
        L.lkv_oracle_get_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: bad argument (rc={rc})")


def row_bytes(bits, D):
    return int(lib().lkv_oracle_row_bytes(bits, D))


def quantize_group(x, bits):
    """Quantize one group of fp32 values; returns (codes uint32, scale, zero)."""
    x = _c(x, np.float32)
    codes = np.zeros(x.shape[0], np.uint32)
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.float32)
    lib().lkv_oracle_quantize_group(_ptr(x), x.shape[0], bits, _ptr(codes), _ptr(s), _ptr(z))
    return codes, s[0], z[0]


def dequant(code, scale, zero):
    return np.float32(lib().lkv_oracle_dequant(int(code), float(scale), float(zero)))


def pack_row(codes, bits):
    codes = _c(codes, np.uint32)
    out = np.zeros(row_bytes(bits, codes.shape[0]), np.uint8)
    lib().lkv_oracle_pack_row(_ptr(codes), codes.shape[0], bits, _ptr(out))
    return out


def unpack_row(row, D, bits):
    row = _c(row, np.uint8)
    out = np.zeros(D, np.uint32)
    lib().lkv_oracle_unpack_row(_ptr(row), D, bits, _ptr(out))
    return out


def dequant_rows(codes, sz, D, G, bits):
    """Dequantize packed rows: codes [..., row_bytes], sz [..., D/G, 2] -> fp32 [..., D]."""
    codes = _c(codes, np.uint8)
    sz = _c(sz, np.float32)
    n = int(np.prod(codes.shape[:-1]))
    out = np.zeros(codes.shape[:-1] + (D,), np.float32)
    _check(lib().lkv_oracle_dequant_rows(_ptr(codes), _ptr(sz), n, D, G, bits, _ptr(out)),
           "dequant_rows")
    return out


def quantize_kv(kb, vb, G, k_bf16, v_bf16, seq_lens):
    """k_bf16, v_bf16: uint16 [B, Hkv, T_cap, D]; returns dict of packed arrays.

    Rows at or beyond a sequence's length are left zero.
    """
    k = _c(k_bf16, np.uint16)
    v = _c(v_bf16, np.uint16)
    sl = _c(seq_lens, np.int32)
    B, Hkv, T_cap, D = k.shape
    ng = D // G
    out = {
        "k_codes": np.zeros((B, Hkv, T_cap, row_bytes(kb, D)), np.uint8),
        "k_sz": np.zeros((B, Hkv, T_cap, ng, 2), np.float32),
        "v_codes": np.zeros((B, Hkv, T_cap, row_bytes(vb, D)), np.uint8),
        "v_sz": np.zeros((B, Hkv, T_cap, ng, 2), np.float32),
    }
    _check(lib().lkv_oracle_quantize_kv(kb, vb, G, B, Hkv, T_cap, D, _ptr(sl), _ptr(k), _ptr(v),
                                        _ptr(out["k_codes"]), _ptr(out["k_sz"]),
                                        _ptr(out["v_codes"]), _ptr(out["v_sz"])), "quantize_kv")
    return out


def decode_attention(kb, vb, G, seq_lens, q_bf16, cache, softmax_scale, tau, want_mask=True,
                     want_p=False):
    """Decode attention over a packed cache; returns (out f32 [B,Hq,D], mask, counts)
    and, with want_p, also p f64 [B, Hq, T_cap].

    mask is u8 [B, Hq, T_cap] (entries t >= T_b stay 0), counts is
    int64 [2] = {skipped (b, h, t) triples, V rows skipped by all heads}.
    """
    q = _c(q_bf16, np.uint16)
    sl = _c(seq_lens, np.int32)
    B, Hq, D = q.shape
    kc = _c(cache["k_codes"], np.uint8)
    Hkv, T_cap = kc.shape[1], kc.shape[2]
    out = np.zeros((B, Hq, D), np.float32)
    mask = np.zeros((B, Hq, T_cap), np.uint8) if want_mask else None
    counts = np.zeros(2, np.int64)
    p = np.zeros((B, Hq, T_cap), np.float64) if want_p else None
    _check(lib().lkv_oracle_decode_attention(
        kb, vb, G, B, Hq, Hkv, T_cap, D, _ptr(sl), _ptr(q), _ptr(kc),
        _ptr(_c(cache["k_sz"], np.float32)), _ptr(_c(cache["v_codes"], np.uint8)),
        _ptr(_c(cache["v_sz"], np.float32)), float(softmax_scale), float(tau), _ptr(out),
        _ptr(mask), _ptr(counts), _ptr(p)), "decode_attention")
    if want_p:
        return out, mask, counts, p
    return out, mask, counts


def attention_mass(p, Hkv, seq_lens):
    """Per-token attention mass of each KV group for the next step's tiers
    ("Super KV Compression" §第二层: the attention weights rank the tokens):
    mass[b, g, t] = mean over the r query heads of group g of p[b, h, t]
    (the softmax probability before the sparse-V skip), for t < T_b; 0 for
    the slots beyond.  p is the f64 [B, Hq, T_cap] of decode_attention."""
    p = np.asarray(p, np.float64)
    B, Hq, T_cap = p.shape
    r = Hq // Hkv
    mass = np.zeros((B, Hkv, T_cap), np.float64)
    for b in range(B):
        T = int(seq_lens[b])
        for g in range(Hkv):
            for h in range(g * r, (g + 1) * r):
                mass[b, g, :T] += p[b, h, :T]
            mass[b, g, :T] /= r
    return mass


def tier_classify(seq_lens, mass, tau_low, tau_high):
    """mass f32 [B, Hkv, T_cap] -> (tier i8, counts i32 [B,Hkv,2], pos2, pos1 i32 [B,Hkv,T_cap]).

    Unused tail entries of pos2 / pos1 are -1 here (the library leaves them unwritten).
    """
    m = _c(mass, np.float32)
    sl = _c(seq_lens, np.int32)
    B, Hkv, T_cap = m.shape
    tier = np.zeros((B, Hkv, T_cap), np.int8)
    counts = np.zeros((B, Hkv, 2), np.int32)
    pos2 = np.full((B, Hkv, T_cap), -1, np.int32)
    pos1 = np.full((B, Hkv, T_cap), -1, np.int32)
    _check(lib().lkv_oracle_tier_classify(B, Hkv, T_cap, _ptr(sl), _ptr(m), float(tau_low),
                                          float(tau_high), _ptr(tier), _ptr(counts),
                                          _ptr(pos2), _ptr(pos1)), "tier_classify")
    return tier, counts, pos2, pos1


def tier_repack(G, k_bf16, v_bf16, counts, pos2, pos1):
    """Quantize kept tokens into segment A (K6, V6) and segment B (K6, V4)."""
    k = _c(k_bf16, np.uint16)
    v = _c(v_bf16, np.uint16)
    B, Hkv, T_cap, D = k.shape
    ng = D // G
    r6, r4 = row_bytes(6, D), row_bytes(4, D)

    def seg(vbits):
        return {"k_codes": np.zeros((B, Hkv, T_cap, r6), np.uint8),
                "k_sz": np.zeros((B, Hkv, T_cap, ng, 2), np.float32),
                "v_codes": np.zeros((B, Hkv, T_cap, r6 if vbits == 6 else r4), np.uint8),
                "v_sz": np.zeros((B, Hkv, T_cap, ng, 2), np.float32)}

    A, Bs = seg(6), seg(4)
    _check(lib().lkv_oracle_tier_repack(
        B, Hkv, T_cap, D, G, _ptr(k), _ptr(v), _ptr(_c(counts, np.int32)),
        _ptr(_c(pos2, np.int32)), _ptr(_c(pos1, np.int32)),
        _ptr(A["k_codes"]), _ptr(A["k_sz"]), _ptr(A["v_codes"]), _ptr(A["v_sz"]),
        _ptr(Bs["k_codes"]), _ptr(Bs["k_sz"]), _ptr(Bs["v_codes"]), _ptr(Bs["v_sz"])),
        "tier_repack")
    return A, Bs


def tiered_attention(G, counts, q_bf16, seg_a, seg_b, softmax_scale, tau, want_p=False):
    """One softmax over the kept tokens of both segments; returns (out, counts)
    and, with want_p, p f64 [B, Hq, T_cap] over segment-A-then-B rows."""
    q = _c(q_bf16, np.uint16)
    B, Hq, D = q.shape
    Hkv, T_cap = seg_a["k_codes"].shape[1], seg_a["k_codes"].shape[2]
    out = np.zeros((B, Hq, D), np.float32)
    sc = np.zeros(2, np.int64)
    p = np.zeros((B, Hq, T_cap), np.float64) if want_p else None
    _check(lib().lkv_oracle_tiered_attention(
        B, Hq, Hkv, T_cap, D, G, _ptr(_c(counts, np.int32)), _ptr(q),
        _ptr(_c(seg_a["k_codes"], np.uint8)), _ptr(_c(seg_a["k_sz"], np.float32)),
        _ptr(_c(seg_a["v_codes"], np.uint8)), _ptr(_c(seg_a["v_sz"], np.float32)),
        _ptr(_c(seg_b["k_codes"], np.uint8)), _ptr(_c(seg_b["k_sz"], np.float32)),
        _ptr(_c(seg_b["v_codes"], np.uint8)), _ptr(_c(seg_b["v_sz"], np.float32)),
        float(softmax_scale), float(tau), _ptr(out), _ptr(sc), _ptr(p)), "tiered_attention")
    if want_p:
        return out, sc, p
    return out, sc


def attention_bf16(seq_lens, q_bf16, k_bf16, v_bf16, softmax_scale):
    """fp64 softmax attention over the unquantized bf16 K/V (raw uint16 bits,
    [B][Hkv][T_cap][D]); q bf16 bits [B][Hq][D].  Returns f32 [B][Hq][D]."""
    B, Hq, D = q_bf16.shape
    Hkv, T_cap = k_bf16.shape[1], k_bf16.shape[2]
    q, k, v = _c(q_bf16, np.uint16), _c(k_bf16, np.uint16), _c(v_bf16, np.uint16)
    out = np.zeros((B, Hq, D), np.float32)
    _check(lib().lkv_oracle_attention_bf16(B, Hq, Hkv, T_cap, D, _ptr(_c(seq_lens, np.int32)), _ptr(q), _ptr(k),
                                           _ptr(v), float(softmax_scale), _ptr(out)), "attention_bf16")
    return out


def set_threads(n):
    """Run the oracle's parallel loops on n threads."""
    lib().lkv_oracle_set_threads(int(n))


def threads():
    """Number of threads the oracle's parallel loops use."""
    return int(lib().lkv_oracle_get_threads())
