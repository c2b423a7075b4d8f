"""The C ABI without a GPU: libhmd.so loads, exports every entry point include/hmd.h declares,
and rejects bad arguments on the host (a status, no launch). These calls never reach a kernel:
validation returns before any CUDA call, so they run on a machine without a GPU.
"""
import ctypes
import os
import re

import pytest

import hybrid_mixer_decoding_b200 as hmd
from hybrid_mixer_decoding_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # a 16-byte aligned non-null address that validation never dereferences
ARG, SHAPE, DTYPE, UNSUP = 1, 2, 3, 6


def _declared():
    with open(os.path.join(ROOT, "include", "hmd.h")) as f:
        src = f.read()
    return re.findall(r"^HMD_API\s+[\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)


def test_library_exports_every_declared_symbol():
    L = hmd.lib()
    names = _declared()
    assert len(names) >= 16
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib._SIGS), "binding and header disagree"


def test_status_strings_and_version():
    assert hmd.hmd_version().startswith("hmd")
    for s in range(8):
        assert hmd.hmd_status_string(s)
    assert hmd.hmd_status_string(99) == "unknown status"


def _decode(kind=hmd.GDN, B=2, H=2, dk=64, dv=64, dtype=hmd.BF16, ptr=FAKE, n_slots=4):
    return hmd.lib().delta_rule_decode(kind, B, H, dk, dv, dtype, ptr, ptr, ptr, ptr, ptr, ptr,
                                       n_slots, None, ptr, 1.0, None)


def test_delta_decode_validation():
    assert _decode(kind=hmd.FA) == ARG
    assert _decode(dtype=7) == DTYPE
    assert _decode(B=-1) == SHAPE
    assert _decode(ptr=None) == ARG
    assert _decode(dk=96) == UNSUP
    assert _decode(dv=6) == UNSUP
    assert _decode(n_slots=1) == SHAPE          # B=2 sequences, no slot map, 1 slot
    assert _decode(B=0) == 0                    # empty batch: nothing to do
    assert hmd.hmd_last_error() == SHAPE        # the last failing status, cleared on read
    assert hmd.hmd_last_error() == 0


def _prefill(kind=hmd.KDA, B=1, T=64, H=1, dk=128, dv=128, dtype=hmd.BF16, chunk=64, ptr=FAKE):
    return hmd.lib().delta_rule_prefill_chunked(kind, B, T, H, dk, dv, dtype, ptr, ptr, ptr, ptr,
                                                ptr, ptr, 4, None, ptr, chunk, 1.0, None)


def test_prefill_validation():
    assert _prefill(kind=hmd.SWA) == ARG
    assert _prefill(chunk=0) == SHAPE
    assert _prefill(chunk=32) == UNSUP
    assert _prefill(dk=200) == UNSUP
    assert _prefill(ptr=None) == ARG
    assert _prefill(T=0) == 0


def _prefill_ws(ws, ws_bytes, B=2, T=300, H=3, dtype=hmd.BF16, dk=128):
    return hmd.lib().delta_rule_prefill_chunked_ws(hmd.GDN, B, T, H, dk, dk, dtype, FAKE, FAKE,
                                                   FAKE, FAKE, FAKE, FAKE, 8, None, FAKE, 64,
                                                   1.0, ws, ws_bytes, None)


def test_prefill_workspace_size_and_validation():
    f = hmd.delta_rule_prefill_workspace_size
    rec = 74240  # Qt, -W, Kc (bf16 64x128), P (bf16 64x64), e^{G_C} (128 fp32), Ut (bf16 64x128)
    assert rec == 4 * 64 * 128 * 2 + 64 * 64 * 2 + 128 * 4
    assert f(hmd.KDA, 4, 4096, 16, 128, 128, hmd.BF16, 64) == 4 * 16 * 64 * rec
    assert f(hmd.GDN, 2, 65, 3, 128, 128, hmd.BF16, 64) == 2 * 3 * 2 * rec   # ragged: 2 chunks
    assert f(hmd.GDN, 2, 65, 3, 64, 64, hmd.BF16, 64) == 0     # CUDA-core path: no scratch
    assert f(hmd.GDN, 2, 65, 3, 128, 128, hmd.F32, 64) == 0
    assert f(hmd.GDN, 0, 65, 3, 128, 128, hmd.BF16, 64) == 0
    one = 2 * 3 * rec                                          # one chunk for all heads
    assert _prefill_ws(None, one) == ARG                       # tensor-core path needs scratch
    assert _prefill_ws(FAKE + 8, one) == ARG                   # not 16-byte aligned
    assert _prefill_ws(FAKE, one - 16) == SHAPE                # not even one chunk fits
    assert _prefill_ws(FAKE, one, T=0) == 0                    # nothing to do


def _attn(kind=hmd.FA, window=0, B=2, Hq=8, Hkv=2, d=128, PT=64, max_pages=4, max_len=256,
          ws=1 << 30, ptr=FAKE, n_pages=16):
    return hmd.lib().attn_decode(kind, window, B, Hq, Hkv, d, PT, ptr, ptr, ptr, ptr, ptr, n_pages,
                                 ptr, max_pages, ptr, max_len, ptr, ptr, ws, None)


def test_attn_validation():
    assert _attn(kind=hmd.KDA) == ARG
    assert _attn(kind=hmd.SWA, window=0) == ARG
    assert _attn(Hq=6, Hkv=4) == SHAPE           # Hq not a multiple of Hkv
    assert _attn(d=96) == UNSUP
    assert _attn(PT=32) == UNSUP
    assert _attn(Hq=64, Hkv=2) == UNSUP          # GQA group of 32 > 16
    assert _attn(max_pages=3) == SHAPE           # table too narrow for 256 tokens
    assert _attn(ws=16) == SHAPE                 # workspace too small
    assert _attn(ptr=None) == ARG


def _verify(kind=hmd.SWA, window=100, ring=2, n_q=4, B=2, Hq=8, Hkv=2, d=128, PT=64, max_pages=4,
            max_len=256, ws=1 << 30, ptr=FAKE, n_pages=16):
    return hmd.lib().attn_verify(kind, window, ring, n_q, B, Hq, Hkv, d, PT, ptr, ptr, ptr, ptr,
                                 ptr, n_pages, ptr, max_pages, ptr, max_len, ptr, ptr, ws, None)


def test_verify_validation():
    assert _verify(n_q=0) == SHAPE
    assert _verify(n_q=5) == UNSUP               # 5 tokens x GQA group 4 > 16 MMA rows
    assert _verify(n_q=4, Hq=16, Hkv=2) == UNSUP  # 4 x 8 > 16
    # a call that passes every check gets misaligned pointers (HMD_ERR_ARG, the last check
    # before the launch), so that none of these calls can launch anything
    MIS = FAKE + 2
    assert _verify(n_q=16, Hq=8, Hkv=8, ptr=MIS) == ARG  # 16 x 1 rows fit
    # SWA ring must hold window + n_q - 1 = 103 positions: 2 pages of 64
    assert _verify(window=128, ring=2) == SHAPE  # 131 positions need 3 pages
    assert _verify(window=128, ring=3, max_pages=3, ptr=MIS) == ARG
    assert _verify(window=128, ring=3, max_pages=2, max_len=256) == SHAPE  # table < ring
    assert _verify(window=128, ring=3, max_pages=2, max_len=100, ptr=MIS) == ARG  # short sequences
    assert _verify(kind=hmd.FA, ring=0, max_pages=3) == SHAPE  # FA table < 256 tokens
    assert _verify(ws=16) == SHAPE
    assert _verify(ptr=None) == ARG
    assert _verify(B=0) == 0
    # one token on the default ring is the decode step's validation
    assert _verify(window=4096, ring=64, n_q=1, max_pages=64, max_len=8192, ptr=MIS) == ARG
    assert _verify(window=4096, ring=64, n_q=2, max_pages=64, max_len=8192) == SHAPE


def test_verify_workspace_is_decode_workspace_times_rows():
    for kind, w in ((hmd.FA, 0), (hmd.SWA, 4096)):
        for n_q in (1, 2, 4):
            v = hmd.attn_verify_workspace_size(kind, w, n_q, 64, 32, 8, 128, 64, 32768)
            d1 = hmd.attn_decode_workspace_size(kind, w, 64, 32, 8, 128, 64, 32768)
            if n_q == 1:
                assert v == d1
            assert v >= 4 * 64 * n_q * 32 * 130


def test_workspace_size_bounds():
    """Partials are one (m, l) pair and one d-vector per query row and key range, with at most
    256 key ranges and never more ranges than 64-token pages."""
    f = hmd.attn_decode_workspace_size
    for kind, w in ((hmd.FA, 0), (hmd.SWA, 4096)):
        for B, Hq, Hkv, d, L in ((32, 32, 8, 128, 8192), (64, 32, 8, 128, 32768), (1, 8, 2, 64, 65),
                                 (3, 8, 2, 128, 300), (16, 32, 8, 128, 1 << 20)):
            n = f(kind, w, B, Hq, Hkv, d, 64, L)
            pages = -(-L // 64) if kind == hmd.FA else min(-(-L // 64), -(-w // 64) + 1)
            s_max = min(256, pages)
            assert 4 * B * Hq * (d + 2) <= n <= 4 * B * Hq * s_max * (d + 2) + 12, (kind, B, L)
            assert (n - 4 * B * Hq * (d + 2) * (n // (4 * B * Hq * (d + 2)))) <= 12


def test_dispatcher_validation():
    io = hmd.DecodeIO(B=1, H=4, Hkv=1, d=128, dtype=hmd.BF16)
    pl = (ctypes.c_int8 * 3)(0, 9, 3)
    L = hmd.lib()
    assert L.mixer_decode_step(pl, 3, 1, ctypes.byref(io), None, None, None, 0, None) == ARG
    assert L.mixer_decode_step(pl, 3, 3, ctypes.byref(io), None, None, None, 0, None) == ARG
    # FA layer with no KV cache registered, GDN layer with no state cache registered
    assert L.mixer_decode_step(pl, 3, 0, ctypes.byref(io), None, None, None, 0, None) == ARG
    assert L.mixer_decode_step(pl, 3, 2, ctypes.byref(io), None, None, None, 0, None) == ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()


def _attn_prefill(kind=hmd.FA, window=0, B=2, T=100, Hq=8, Hkv=2, d=128, pt=64, n_pages=8,
                  max_pages=2, ptr=FAKE):
    return hmd.lib().attn_prefill(kind, window, B, T, Hq, Hkv, d, pt, ptr, ptr, ptr, ptr, ptr,
                                  n_pages, ptr, max_pages, ptr, None)


def test_attn_prefill_validation():
    assert _attn_prefill(kind=hmd.GDN) == ARG
    assert _attn_prefill(kind=hmd.SWA, window=0) == ARG
    assert _attn_prefill(Hq=6, Hkv=4) == SHAPE          # Hq not a multiple of Hkv
    assert _attn_prefill(Hq=24, Hkv=8) == UNSUP         # group of 3
    assert _attn_prefill(d=96) == UNSUP
    assert _attn_prefill(pt=32) == UNSUP
    assert _attn_prefill(max_pages=1) == SHAPE          # 100 tokens need 2 pages
    assert _attn_prefill(kind=hmd.SWA, window=200, max_pages=3) == SHAPE  # ring of 4 pages
    assert _attn_prefill(ptr=None) == ARG
    assert _attn_prefill(T=0) == 0 and _attn_prefill(B=0) == 0


def test_fused_activation_validation():
    L = hmd.lib()
    from hybrid_mixer_decoding_b200._lib import DeltaAct
    good = DeltaAct(FAKE, FAKE, 1e-6)
    dec = lambda act, B=2, dtype=hmd.BF16: L.delta_rule_decode_act(  # noqa: E731
        hmd.GDN, B, 2, 64, 64, dtype, FAKE, FAKE, FAKE, FAKE, FAKE, act, FAKE, 4, None, None,
        FAKE, 1.0, None)
    assert dec(None) == ARG
    assert dec(ctypes.byref(DeltaAct(None, FAKE, 1e-6))) == ARG
    assert dec(ctypes.byref(DeltaAct(FAKE, None, 1e-6))) == ARG
    assert dec(ctypes.byref(DeltaAct(FAKE, FAKE, -1.0))) == ARG
    assert dec(ctypes.byref(good), B=0) == 0
    pre = lambda act, dtype=hmd.BF16, dk=128: L.delta_rule_prefill_chunked_act(  # noqa: E731
        hmd.KDA, 1, 64, 1, dk, dk, dtype, FAKE, FAKE, FAKE, FAKE, FAKE, act, FAKE, 1, None, FAKE,
        64, 1.0, None)
    assert pre(None) == ARG
    assert pre(ctypes.byref(good), dtype=hmd.F32) == UNSUP   # fused only on the tensor-core path
    assert pre(ctypes.byref(good), dk=64) == UNSUP


def test_prefill_with_prefix_validation():
    """Calls that pass every check get a misaligned output pointer, the last check before the
    launch (HMD_ERR_ARG), so that none of them can launch anything."""
    L = hmd.lib()
    MIS = FAKE + 2
    ext = lambda d=128, max_prefix=128, max_pages=8, T=64, kind=hmd.FA, w=0, pre=FAKE, o=MIS: (  # noqa: E731
        L.attn_prefill_ext(kind, w, 2, T, 8, 2, d, 64, FAKE, FAKE, FAKE, pre, max_prefix, FAKE,
                           FAKE, 16, FAKE, max_pages, o, None))
    assert ext() == ARG                        # every shape check passes
    assert ext(d=64) == ARG                    # d = 64 takes a cached prefix too
    assert ext(d=64, pre=None) == ARG
    assert ext(d=96) == UNSUP
    assert ext(max_prefix=100) == SHAPE        # not a whole number of pages
    assert ext(max_prefix=512, max_pages=8) == SHAPE  # FA table < (512 + 64) / 64 = 9 pages
    assert ext(max_prefix=448, max_pages=8) == ARG
    assert ext(max_prefix=-64) == SHAPE
    assert ext(T=0) == 0


def test_state_cache_save_validation():
    L = hmd.lib()
    ids = (ctypes.c_int32 * 1)(0)
    assert L.state_cache_save(None, 0, ids, 1, FAKE, None) == ARG


def test_header_is_c99_and_links_from_c(tmp_path):
    """include/hmd.h compiles as strict C99, and a C program links against libhmd.so and calls
    it (host-side calls only: version string, status strings, argument validation)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_hmd.c"
    src.write_text(r"""
#include "hmd.h"
#include <stdio.h>
#include <string.h>
int main(void) {
    if (strncmp(hmd_version(), "hmd", 3) != 0) return 1;
    if (strcmp(hmd_status_string(HMD_OK), "ok") != 0) return 2;
    /* a bad kind is rejected on the host, before any device work */
    if (delta_rule_decode((hmd_kind_t)7, 1, 1, 64, 64, HMD_BF16, 0, 0, 0, 0, 0, 0, 1, 0, 0, 1.f,
                          0) != HMD_ERR_ARG) return 3;
    if (hmd_last_error() != HMD_ERR_ARG) return 4;
    printf("ok\n");
    return 0;
}
""")
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    exe = tmp_path / "use_hmd"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-L", lib_dir, "-lhmd",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "ok"


def test_device_error_bits_match_the_header():
    text = open(os.path.join(ROOT, "include", "hmd.h")).read()
    bits = {m.group(1): int(m.group(2), 16)
            for m in re.finditer(r"#define HMD_DEVERR_(\w+)\s+0x([0-9a-fA-F]+)u", text)}
    assert bits == {"TIMEOUT": hmd.DEVERR_TIMEOUT, "PAGE": hmd.DEVERR_PAGE,
                    "SLOT": hmd.DEVERR_SLOT, "SEQLEN": hmd.DEVERR_SEQLEN,
                    "GATE": hmd.DEVERR_GATE}


def test_copy_skip_hook_validation():
    """The failure-detection hook rejects bad arguments on the host; a valid arming launches
    nothing by itself."""
    L = hmd.lib()
    hmd.hmd_last_error()
    assert L.hmd_test_arm_copy_skip(7, 0, 10**6) == ARG          # no such kernel
    assert L.hmd_test_arm_copy_skip(_lib.TEST_DELTA_DECODE, -2, 10**6) == ARG
    assert L.hmd_test_arm_copy_skip(_lib.TEST_ATTN_SPLIT, 0, 10) == ARG        # below 1 us
    assert L.hmd_test_arm_copy_skip(_lib.TEST_ATTN_SPLIT, 0, 3 * 10**9) == ARG  # above 2 s
    assert hmd.hmd_last_error() == ARG
    assert L.hmd_test_arm_copy_skip(_lib.TEST_DELTA_DECODE, 3, 10**6) == 0
    # a call rejected on the host leaves the fault armed and launches nothing; cta = -1 disarms
    # it, so no later test in this thread meets it
    assert _decode(ptr=None) == ARG
    assert L.hmd_test_arm_copy_skip(_lib.TEST_DELTA_DECODE, -1, 10**6) == 0
