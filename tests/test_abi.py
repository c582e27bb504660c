"""The C ABI, without a GPU: liblkv.so loads, exports every entry point that
include/lkv.h declares, and rejects bad arguments on the host before it
launches anything (fake device addresses are never dereferenced)."""
import os
import re

import pytest

from quantized_kv_cache_lkv_b200 import lkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lkv.h")

FAKE = 0x7F0000000000        # 16-byte aligned, never dereferenced
MISALIGNED = FAKE + 8
K6V4 = (6, 4, 64)


@pytest.fixture(scope="module")
def L():
    from quantized_kv_cache_lkv_b200 import build
    build.build()
    return lkv.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^LKV_API\s+[\w\s\*]+?\b(lkv_\w+)\s*\(", text, re.M)))


def test_header_declarations_are_all_exported(L):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    # the binding wraps exactly the declared set
    assert sorted(lkv.SIGNATURES) == names


def test_status_strings_and_sizes(L):
    assert lkv.lkv_status_string(0) == "LKV_OK"
    assert lkv.lkv_status_string(5) == "LKV_ERR_TIMEOUT"
    assert lkv.lkv_status_string(99) == "LKV_ERR_UNKNOWN"
    assert lkv.lkv_version() == 100
    assert lkv.lkv_row_bytes(6, 128) == 96 and lkv.lkv_row_bytes(4, 128) == 64
    assert lkv.lkv_row_bytes(2, 64) == 16 and lkv.lkv_row_bytes(8, 64) == 64
    assert lkv.lkv_row_bytes(5, 128) == 0
    assert lkv.lkv_sz_row_bytes(128, 64) == 16 and lkv.lkv_sz_row_bytes(64, 32) == 16
    assert lkv.lkv_sz_row_bytes(64, 128) == 0


def test_workspace_sizes(L):
    # groups of up to 4 query heads: single-launch decode (logits in an L2-resident workspace)
    n = lkv.lkv_decode_workspace_bytes(K6V4, 16, 32, 8, 8192, 128)
    assert 16 * 8 * 8192 * 4 * 4 <= n < 64 << 20 and n % 256 == 0
    # larger groups: three-launch decode, logits in the workspace
    n8 = lkv.lkv_decode_workspace_bytes(K6V4, 16, 64, 8, 8192, 128)
    logits = 16 * 8 * 8192 * 8 * 4
    assert logits < n8 < logits * 2
    assert lkv.lkv_decode_workspace_bytes(K6V4, 16, 30, 8, 8192, 128) == 0   # Hq % Hkv
    assert lkv.lkv_decode_workspace_bytes((5, 4, 64), 1, 4, 2, 256, 64) == 0
    assert lkv.lkv_tiered_workspace_bytes(32, 32, 8, 32768, 128, 64) > 0


def rc_of(fn, *args, **kwargs):
    try:
        fn(*args, **kwargs)
    except lkv.LkvError as e:
        return e.status
    return 0


def quant_args(**kw):
    a = dict(spec=K6V4, B=2, Hkv=2, T_cap=64, D=128, seq_lens=FAKE, k=FAKE, v=FAKE, k_codes=FAKE,
             k_sz=FAKE, v_codes=FAKE, v_sz=FAKE, stream=0)
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,want", [
    (dict(spec=(5, 4, 64)), lkv.LKV_ERR_UNSUPPORTED),
    (dict(spec=(6, 4, 48)), lkv.LKV_ERR_UNSUPPORTED),
    (dict(spec=(6, 4, 256)), lkv.LKV_ERR_UNSUPPORTED),
    (dict(D=96), lkv.LKV_ERR_UNSUPPORTED),
    (dict(spec=(6, 4, 128), T_cap=63), lkv.LKV_ERR_UNSUPPORTED),   # T_cap * ng odd
    (dict(B=-1), lkv.LKV_ERR_INVALID_ARG),
    (dict(Hkv=0), lkv.LKV_ERR_INVALID_ARG),
    (dict(k=None), lkv.LKV_ERR_INVALID_ARG),
    (dict(v_sz=MISALIGNED), lkv.LKV_ERR_INVALID_ARG),
    (dict(seq_lens=None), lkv.LKV_ERR_INVALID_ARG),
])
def test_quantize_rejects(L, kw, want):
    assert rc_of(lambda **a: lkv.lkv_quantize_kv(**a), **quant_args(**kw)) == want


def test_empty_inputs_are_no_ops(L):
    # nothing to do: succeeds without touching any pointer or the GPU
    assert rc_of(lambda **a: lkv.lkv_quantize_kv(**a), **quant_args(B=0, k=None, v=None)) == 0
    assert rc_of(lambda **a: lkv.lkv_quantize_kv(**a), **quant_args(T_cap=0)) == 0
    assert rc_of(lkv.lkv_tier_classify, 0, 8, 64, None, None, 0.0, 1.0, None, None, None, None, 0) == 0


def decode_args(**kw):
    a = dict(spec=K6V4, B=2, Hq=8, Hkv=2, T_cap=64, D=128, seq_lens=FAKE, q=FAKE, k_codes=FAKE,
             k_sz=FAKE, v_codes=FAKE, v_sz=FAKE, softmax_scale=0.088, tau=0.0, out=FAKE,
             skip_mask=None, skip_counts=None, workspace=FAKE, ws_bytes=1 << 40, stream=0)
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,want", [
    (dict(Hq=7), lkv.LKV_ERR_INVALID_ARG),
    (dict(Hq=6), lkv.LKV_ERR_UNSUPPORTED),                    # r = 3
    (dict(Hq=256, Hkv=2), lkv.LKV_ERR_UNSUPPORTED),           # r > 64
    (dict(D=256), lkv.LKV_ERR_UNSUPPORTED),
    (dict(spec=(6, 3, 64)), lkv.LKV_ERR_UNSUPPORTED),
    (dict(softmax_scale=float("inf")), lkv.LKV_ERR_INVALID_ARG),
    (dict(tau=float("nan")), lkv.LKV_ERR_INVALID_ARG),
    (dict(q=None), lkv.LKV_ERR_INVALID_ARG),
    (dict(out=MISALIGNED), lkv.LKV_ERR_INVALID_ARG),
    (dict(skip_counts=MISALIGNED), lkv.LKV_ERR_INVALID_ARG),
    (dict(workspace=None), lkv.LKV_ERR_INVALID_ARG),
    (dict(workspace=FAKE + 16), lkv.LKV_ERR_INVALID_ARG),     # not 256-byte aligned
    (dict(ws_bytes=1024), lkv.LKV_ERR_WORKSPACE),
])
def test_decode_rejects(L, kw, want):
    assert rc_of(lambda **a: lkv.lkv_decode_attention(**a), **decode_args(**kw)) == want


def test_static_decode_rejects_before_any_device_call(L):
    """The fixed-scratch decode refuses sizes beyond its scratch on the host."""
    def static_args(**kw):
        a = decode_args(status=None)
        del a["workspace"], a["ws_bytes"]
        a.update(kw)
        return a
    call = lambda **a: lkv.lkv_decode_attention_static(**a)
    # B64 x 8 kv heads x T4096 needs about 40 MiB of scratch
    assert lkv.lkv_decode_workspace_bytes(K6V4, 64, 32, 8, 4096, 128) > lkv.LKV_STATIC_WORKSPACE_BYTES
    assert rc_of(call, **static_args(B=64, Hq=32, Hkv=8, T_cap=4096)) == lkv.LKV_ERR_WORKSPACE
    assert rc_of(call, **static_args(status=FAKE + 2)) == lkv.LKV_ERR_INVALID_ARG
    assert rc_of(call, **static_args(Hq=6)) == lkv.LKV_ERR_UNSUPPORTED
    assert rc_of(call, **static_args(q=None)) == lkv.LKV_ERR_INVALID_ARG


def test_append_and_mass_reject(L):
    call = lambda *a: lkv.lkv_append_kv(*a)
    base = [K6V4, 2, 2, 64, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0]
    assert rc_of(call, (5, 4, 64), *base[1:]) == lkv.LKV_ERR_UNSUPPORTED
    assert rc_of(call, *base[:5], None, *base[6:]) == lkv.LKV_ERR_INVALID_ARG      # pos
    assert rc_of(call, *base[:6], MISALIGNED, *base[7:]) == lkv.LKV_ERR_INVALID_ARG
    assert rc_of(call, K6V4, 0, 2, 64, 128, None, None, None, None, None, None, None, 0) == 0   # nothing to do
    m = decode_args()
    del m["workspace"], m["ws_bytes"]
    mass = lambda **kw: lkv.lkv_decode_attention_mass(**dict(m, **kw))
    assert rc_of(mass, mass=None, workspace=FAKE, ws_bytes=1 << 40) == lkv.LKV_ERR_INVALID_ARG
    assert rc_of(mass, mass=FAKE + 2, workspace=FAKE, ws_bytes=1 << 40) == lkv.LKV_ERR_INVALID_ARG
    assert rc_of(mass, mass=FAKE, workspace=FAKE, ws_bytes=64) == lkv.LKV_ERR_WORKSPACE


def test_paged_rejects(L):
    pq = [K6V4, 2, 2, 3, 8, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0]
    assert rc_of(lkv.lkv_quantize_kv_paged, *pq[:3], 0, *pq[4:]) == lkv.LKV_ERR_INVALID_ARG       # pages_per_seq
    assert rc_of(lkv.lkv_quantize_kv_paged, *pq[:4], 0, *pq[5:]) == lkv.LKV_ERR_INVALID_ARG       # num_pages
    assert rc_of(lkv.lkv_quantize_kv_paged, *pq[:9], None, *pq[10:]) == lkv.LKV_ERR_INVALID_ARG   # table
    assert rc_of(lkv.lkv_append_kv_paged, *pq[:9], None, *pq[10:]) == lkv.LKV_ERR_INVALID_ARG
    pd = [K6V4, 2, 16, 2, 3, 8, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.088, 0.0, FAKE, None, None,
          FAKE, 1 << 40, 0]
    assert rc_of(lkv.lkv_decode_attention_paged, *pd) == lkv.LKV_ERR_UNSUPPORTED                # groups of 8
    pd[2] = 8
    assert rc_of(lkv.lkv_decode_attention_paged, *pd[:9], None, *pd[10:]) == lkv.LKV_ERR_INVALID_ARG
    assert rc_of(lkv.lkv_decode_attention_paged, *pd[:20], 64, pd[21]) == lkv.LKV_ERR_WORKSPACE


def test_tiered_rejects(L):
    seg = lkv.lkv_segment(FAKE, FAKE, FAKE, FAKE)
    bad = lkv.lkv_segment(FAKE, None, FAKE, FAKE)
    base = [2, 8, 2, 64, 128, 64, FAKE, FAKE]
    assert rc_of(lkv.lkv_tiered_attention, *base, seg, bad, 0.088, 0.0, FAKE, None, FAKE, 1 << 40, 0) \
        == lkv.LKV_ERR_INVALID_ARG
    assert rc_of(lkv.lkv_tiered_attention, *base, seg, seg, 0.088, 0.0, FAKE, None, FAKE, 64, 0) \
        == lkv.LKV_ERR_WORKSPACE
    assert rc_of(lkv.lkv_tier_repack, 2, 2, 64, 128, 48, FAKE, FAKE, FAKE, FAKE, FAKE, seg, seg, 0) \
        == lkv.LKV_ERR_UNSUPPORTED
    assert rc_of(lkv.lkv_tier_classify, 2, 0, 64, FAKE, FAKE, 0.0, 1.0, FAKE, FAKE, FAKE, FAKE, 0) \
        == lkv.LKV_ERR_INVALID_ARG
    # the composite call validates all three stages before enqueueing any
    assert rc_of(lkv.lkv_tiered_decode, 2, 8, 2, 64, 128, 64, FAKE, FAKE, 1e-4, 1e-2, FAKE, FAKE, FAKE,
                 FAKE, FAKE, FAKE, None, seg, seg, 0.088, 0.0, FAKE, None, FAKE, 1 << 40, 0) \
        == lkv.LKV_ERR_INVALID_ARG


def test_binding_raises_without_library(monkeypatch, tmp_path):
    """No fallback: with the shared library absent every call raises."""
    monkeypatch.setattr(lkv, "_lib", None)
    monkeypatch.setattr(lkv, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        lkv.lkv_version()


def test_plain_c_client(L, tmp_path):
    """A C11 program that includes only include/lkv.h compiles with gcc
    (-Wall -Werror), links liblkv.so and gets the documented results of the
    calls that need no GPU: the boundary is usable from plain C."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    pkg = os.path.dirname(lkv.LIB_PATH)
    exe = tmp_path / "abi_client"
    build = subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "abi_client.c"), "-L", pkg, "-llkv",
                            f"-Wl,-rpath,{pkg}", "-o", str(exe)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
