"""Device buffers for liblkv calls, allocated with torch (memory plumbing only).

Shapes follow include/lkv.h: codes u8 [B][Hkv][T_cap][D*bits/8], (scale, zero)
f32 [B][Hkv][T_cap][D/G][2], tiers i8 / counts i32 / positions i32.
"""
import torch


def alloc_cache(k_bits, v_bits, G, B, Hkv, T_cap, D, device="cuda", zero=False):
    mk = torch.zeros if zero else torch.empty
    ng = D // G
    return {
        "k_codes": mk(B, Hkv, T_cap, D * k_bits // 8, dtype=torch.uint8, device=device),
        "k_sz": mk(B, Hkv, T_cap, ng, 2, dtype=torch.float32, device=device),
        "v_codes": mk(B, Hkv, T_cap, D * v_bits // 8, dtype=torch.uint8, device=device),
        "v_sz": mk(B, Hkv, T_cap, ng, 2, dtype=torch.float32, device=device),
    }


def alloc_segments(G, B, Hkv, T_cap, D, device="cuda", zero=False):
    """Segment A (K6, V6) and segment B (K6, V4) of the tiered cache."""
    return (alloc_cache(6, 6, G, B, Hkv, T_cap, D, device, zero),
            alloc_cache(6, 4, G, B, Hkv, T_cap, D, device, zero))


def alloc_tiers(B, Hkv, T_cap, device="cuda", zero=False):
    mk = torch.zeros if zero else torch.empty
    return {
        "tier": mk(B, Hkv, T_cap, dtype=torch.int8, device=device),
        "counts": mk(B, Hkv, 2, dtype=torch.int32, device=device),
        "pos_a": mk(B, Hkv, T_cap, dtype=torch.int32, device=device),
        "pos_b": mk(B, Hkv, T_cap, dtype=torch.int32, device=device),
    }


def alloc_workspace(n_bytes, device="cuda"):
    """A zero-filled workspace (the state every liblkv call expects on first use)."""
    return torch.zeros(max(int(n_bytes), 256), dtype=torch.uint8, device=device)
