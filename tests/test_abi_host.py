"""The C-ABI library without a GPU: it builds, loads, exports every declared symbol, and
rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "binattn.h")


@pytest.fixture(scope="module")
def L():
    from bit_qk_attention_b200 import build
    import bit_qk_attention_b200 as ba
    build.build()
    return ba.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ba_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("ba_pack_signs", "ba_quant_v", "ba_attention_fwd", "ba_attention_fwd_packed"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    from bit_qk_attention_b200 import LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (ba_\w+)$", out.stdout, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        getattr(L, n)  # resolvable through ctypes


def test_binding_covers_every_symbol():
    import bit_qk_attention_b200 as ba
    assert set(declared_functions()) == set(ba.SIGNATURES)


def test_host_queries(L):
    assert L.ba_sign_words(1) == 4 and L.ba_sign_words(128) == 4
    assert L.ba_sign_words(0) == 0 and L.ba_sign_words(129) == 0
    assert [L.ba_v_row_bytes(d) for d in (1, 16, 17, 64, 72, 128)] == [16, 16, 32, 64, 80, 128]
    assert L.ba_kv_block() == 128
    # one-launch preparation: many short slices of whole 16-byte rows
    assert L.ba_prep_fused(64, 12, 197, 64) == 1 and L.ba_prep_fused(32, 16, 256, 72) == 1
    assert L.ba_prep_fused(1, 16, 4096, 64) == 0 and L.ba_prep_fused(64, 12, 197, 60) == 0
    assert L.ba_prep_fused(64, 12, 197, 16) == 0 and L.ba_prep_fused(0, 12, 197, 64) == 0
    assert L.ba_prep_fused(64, 12, 197, 129) == 0
    # one launch while a slice fits in two batches of 10 passes: 2 * 10 * (256 / (d/8)) rows
    assert L.ba_prep_fused(8, 16, 640, 64) == 1 and L.ba_prep_fused(8, 16, 641, 64) == 0
    assert L.ba_workspace_bytes(0, 4, 16, 64) == 0 and L.ba_workspace_bytes(2, 4, 0, 64) == 0
    big = L.ba_workspace_bytes(2, 16, 4096, 64)
    assert big >= 2 * 16 * 4096 * (16 + 16 + 64)
    assert L.ba_workspace_bytes(2, 16, 4096, 129) == ctypes.c_size_t(-1).value
    assert L.ba_pack_workspace_bytes(2, 16, 4096, 64) < big and L.ba_quant_workspace_bytes(2, 16, 4096, 64) < big
    for s in range(7):
        assert L.ba_status_string(s).startswith(b"BA_")


def test_p_code_thresholds(L):
    """The tcgen05 kernel's exact-code thresholds against the definition's P code of
    d = s - m, written out here: code(d) = min(255, rne(fl32(255 * fl32(exp(d))))). Each
    threshold is the least double whose code exceeds k: its code is at least k + 1, and the next
    double below it has a code of at most k."""
    import math
    import numpy as np

    def code(d):
        p = np.float32(math.exp(d))
        return int(min(np.rint(np.float32(255.0) * p), 255.0))

    prev = -math.inf
    for k in range(255):
        t = L.ba_p_code_threshold(k)
        assert prev < t < 0.0
        assert code(t) >= k + 1
        assert code(math.nextafter(t, -math.inf)) <= k
        # the real boundary 255 exp(d) = k + 1/2, moved only by the two fp32 roundings
        assert abs(t - math.log((k + 0.5) / 255.0)) < 1e-6
        prev = t
    assert math.isnan(L.ba_p_code_threshold(255)) and math.isnan(L.ba_p_code_threshold(-1))


def test_noalloc_limit_matches_header():
    import bit_qk_attention_b200 as ba
    text = open(HEADER).read()
    m = re.search(r"#define BA_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", text)
    assert m, "BA_NOALLOC_SCRATCH_BYTES not found"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == ba.NOALLOC_SCRATCH_BYTES


def test_impl_switch(L):
    assert L.ba_set_attention_impl(3) == 1
    assert L.ba_set_attention_impl(1) == 0 and L.ba_get_attention_impl() == 1
    assert L.ba_set_attention_impl(0) == 0 and L.ba_get_attention_impl() == 0


def test_empty_problems_launch_nothing(L):
    import bit_qk_attention_b200 as ba
    nb = ba.CBias()
    for (B, H, N) in ((0, 4, 16), (2, 0, 16), (2, 4, 0)):
        assert L.ba_attention_fwd(None, None, None, 0, B, H, N, 64, ctypes.byref(nb), 0.0, None, 2, None, 0,
                                  None, None) == 0
        assert L.ba_pack_signs(None, 0, B, H, N, 64, None, None, None, 0, None) == 0
        assert L.ba_quant_v(None, 1, B, H, N, 64, None, None, None, 0, None) == 0


# The cases below pass fake device addresses: each must be rejected by the host-side
# checks. They only run where no GPU is present, so nothing can ever reach a device.
no_gpu = pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="fake pointers: host-only")

FAKE = 0x10000


@no_gpu
def test_forward_argument_errors(L):
    import bit_qk_attention_b200 as ba
    nb = ba.CBias()
    ws_need = L.ba_workspace_bytes(2, 3, 40, 64)

    def call(q=FAKE, k=FAKE, v=FAKE, dt=0, B=2, H=3, N=40, d=64, bias=nb, scale=0.0, o=FAKE, odt=2, ws=FAKE,
             nws=ws_need, dbg=None):
        return L.ba_attention_fwd(q, k, v, dt, B, H, N, d, ctypes.byref(bias), scale, o, odt, ws, nws, dbg, None)

    assert call(d=0) == 2 and call(d=129) == 2
    assert call(B=-1) == 1 and call(N=-5) == 1
    assert call(B=300, H=300) == 2 and call(N=(1 << 20) + 1) == 2
    assert call(dt=2) == 1 and call(dt=7) == 1 and call(odt=9) == 1
    assert call(scale=float("nan")) == 1 and call(scale=float("inf")) == 1
    assert call(q=None) == 1 and call(v=None) == 1 and call(o=None) == 1
    assert call(q=FAKE + 8) == 3 and call(o=FAKE + 2) == 3 and call(dbg=FAKE + 4) == 3
    assert call(ws=None) == 4 and call(nws=ws_need - 1) == 4 and call(ws=FAKE + 8) == 3
    bad = ba.CBias(7, FAKE, 0, 0, 0, 0, 0, 0)
    assert call(bias=bad) == 1
    assert call(bias=ba.CBias(1, None, 0, 0, 0, 0, 0, 0)) == 1
    assert call(bias=ba.CBias(1, FAKE + 4, 0, 0, 0, 0, 0, 0)) == 3
    assert call(bias=ba.CBias(1, FAKE, -1, 0, 0, 0, 0, 0)) == 1
    assert call(bias=ba.CBias(2, FAKE, 0, 5, 8, 5, 8, 0), nws=ws_need - 1) == 4  # valid bias, then ws
    assert call(bias=ba.CBias(2, FAKE, 0, 5, 8, 5, 8, 1)) == 1  # 5*8 != 40 - 1
    assert call(bias=ba.CBias(2, FAKE, 0, 5, 8, 4, 8, 0)) == 1  # table smaller than the grid
    assert call(bias=ba.CBias(2, FAKE, 0, 0, 40, 1, 40, 0)) == 1


@no_gpu
def test_step_argument_errors(L):
    need = L.ba_pack_workspace_bytes(1, 2, 50, 72)
    assert L.ba_pack_signs(FAKE, 0, 1, 2, 50, 72, FAKE, FAKE, FAKE, need - 1, None) == 4
    assert L.ba_pack_signs(FAKE, 2, 1, 2, 50, 72, FAKE, FAKE, FAKE, need, None) == 1
    assert L.ba_pack_signs(FAKE, 0, 1, 2, 50, 72, FAKE + 4, FAKE, FAKE, need, None) == 3
    assert L.ba_pack_signs(None, 0, 1, 2, 50, 72, FAKE, FAKE, FAKE, need, None) == 1
    needq = L.ba_quant_workspace_bytes(1, 2, 50, 72)
    assert L.ba_quant_v(FAKE, 1, 1, 2, 50, 72, FAKE, FAKE, None, needq, None) == 4
    assert L.ba_quant_v(FAKE, 1, 1, 2, 50, 72, FAKE, None, FAKE, needq, None) == 1
    nb = __import__("bit_qk_attention_b200").CBias()
    assert L.ba_attention_fwd_packed(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 2, 50, 72, ctypes.byref(nb), 0.0,
                                     FAKE, 2, None, None) == 1
    assert L.ba_attention_fwd_packed(FAKE, FAKE, FAKE, FAKE + 4, FAKE, FAKE, 1, 2, 50, 72, ctypes.byref(nb),
                                     0.0, FAKE, 2, None, None) == 3
    assert L.ba_attention_fwd_packed(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 50, 72, ctypes.byref(nb), 0.0,
                                     FAKE, 5, None, None) == 1
