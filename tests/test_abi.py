"""CPU-side checks of the C ABI: the library loads, exports every function the header
declares, and rejects bad arguments on the host before launching anything.  No call here
reaches a kernel: each one either fails validation or has no work (R = 0 / T = 0), so the
suite runs without a GPU."""
import ctypes
import os

import pytest

from linear_attention_diffusion_hedgehog_b200 import bha

P = ctypes.c_void_p
A16 = P(0x10000)      # a 16-byte-aligned fake device address (never dereferenced on the host)
A16b = P(0x20000)
A16c = P(0x30000)
MIS = P(0x10004)      # 4-byte aligned, not 16-byte aligned
NULL = None


def dims(**kw):
    base = dict(R=4, Hq=16, Hkv=4, d=128, F=256, max_block=32, T=128, num_slots=4, act_dtype=0)
    base.update(kw)
    return bha.make_dims(base["R"], base["Hq"], base["Hkv"], base["d"], base["F"],
                         base["max_block"], base["T"], base["num_slots"], base["act_dtype"])


def hybrid(dm, cu=A16, slot=NULL, Q=A16, K=A16b, V=A16c, S=P(0x40000), Z=P(0x50000),
           W=P(0x60000), alpha=NULL, O=P(0x70000), err=NULL):
    return bha.lib().bha_hybrid_attn(ctypes.byref(dm), cu, slot, Q, K, V, S, Z, W, alpha, O, err,
                                     NULL)


def commit(dm, cu=A16, slot=NULL, K=A16, V=A16b, W=A16c, S=P(0x40000), Z=P(0x50000), err=NULL):
    return bha.lib().bha_commit_block(ctypes.byref(dm), cu, slot, K, V, W, S, Z, err, NULL)


def test_library_exports_every_header_function():
    names = bha.header_functions()
    assert {"bha_featuremap", "bha_hybrid_attn", "bha_commit_block", "bha_full_prefix_attn",
            "bha_status_string"} <= set(names)
    L = bha.lib()
    for n in names:
        assert hasattr(L, n), f"libbha.so does not export {n}"


def test_version_and_status_strings():
    assert bha.lib().bha_version() >= 100
    for code in (0, -1, -2, -3, -4):
        assert bha.status_string(code).startswith("BHA_")
    assert "unknown" in bha.status_string(7)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), bha.BHA_ERR_INVALID),          # Hq % Hkv != 0
    (dict(F=255), bha.BHA_ERR_INVALID),                # odd F
    (dict(R=-1), bha.BHA_ERR_INVALID),
    (dict(max_block=0), bha.BHA_ERR_INVALID),
    (dict(max_block=129), bha.BHA_ERR_UNSUPPORTED),    # block longer than the kernels take
    (dict(d=257), bha.BHA_ERR_UNSUPPORTED),
    (dict(F=514), bha.BHA_ERR_UNSUPPORTED),
    (dict(act_dtype=5), bha.BHA_ERR_INVALID),
    (dict(num_slots=3), bha.BHA_ERR_INVALID),          # identity slots need num_slots >= R
])
def test_bad_dims_are_rejected(kw, code):
    assert hybrid(dims(**kw)) == code


def test_null_dims():
    assert bha.lib().bha_hybrid_attn(None, A16, NULL, A16, A16, A16, A16, A16, A16, NULL, A16b,
                                     NULL, NULL) == bha.BHA_ERR_INVALID


@pytest.mark.parametrize("arg", ["cu", "Q", "K", "V", "S", "Z", "W", "O"])
def test_null_pointer_is_rejected(arg):
    assert hybrid(dims(), **{arg: NULL}) == bha.BHA_ERR_INVALID


@pytest.mark.parametrize("arg", ["Q", "K", "V", "S", "Z", "W", "O"])
def test_misaligned_tensor_is_rejected(arg):
    assert hybrid(dims(), **{arg: MIS}) == bha.BHA_ERR_INVALID


def test_aliased_output_is_rejected():
    assert hybrid(dims(), O=A16) == bha.BHA_ERR_INVALID  # O == Q


def test_no_work_returns_ok_without_launch():
    assert hybrid(dims(R=0), cu=NULL, Q=NULL) == bha.BHA_OK
    assert hybrid(dims(T=0)) == bha.BHA_OK
    assert commit(dims(R=0), cu=NULL) == bha.BHA_OK


def test_commit_validation():
    assert commit(dims(), S=MIS) == bha.BHA_ERR_INVALID
    assert commit(dims(), K=NULL) == bha.BHA_ERR_INVALID
    assert commit(dims(), Z=P(0x40000)) == bha.BHA_ERR_INVALID  # S aliases Z
    assert commit(dims(Hq=3, Hkv=2)) == bha.BHA_ERR_INVALID


def test_featuremap_validation():
    L = bha.lib()
    dm = dims()
    assert L.bha_featuremap(ctypes.byref(dm), A16, 0, A16b, A16c, 0, NULL) == bha.BHA_ERR_INVALID
    assert L.bha_featuremap(ctypes.byref(dm), A16, 4, A16b, A16c, 9, NULL) == bha.BHA_ERR_INVALID
    assert L.bha_featuremap(ctypes.byref(dm), MIS, 4, A16b, A16c, 0, NULL) == bha.BHA_ERR_INVALID
    assert L.bha_featuremap(ctypes.byref(dm), A16, 4, A16b, A16, 0, NULL) == bha.BHA_ERR_INVALID
    assert L.bha_featuremap(ctypes.byref(dims(T=0)), A16, 4, A16b, A16c, 0, NULL) == bha.BHA_OK
    # the checked form validates the same way, plus a misaligned error word
    assert L.bha_featuremap_checked(ctypes.byref(dm), A16, 0, A16b, A16c, 0, NULL, NULL) == bha.BHA_ERR_INVALID
    assert L.bha_featuremap_checked(ctypes.byref(dm), MIS, 4, A16b, A16c, 0, NULL, NULL) == bha.BHA_ERR_INVALID
    assert L.bha_featuremap_checked(ctypes.byref(dm), A16, 4, A16b, A16c, 0, P(0x20001), NULL) == bha.BHA_ERR_INVALID
    assert L.bha_featuremap_checked(ctypes.byref(dims(T=0)), A16, 4, A16b, A16c, 0, P(0x20000), NULL) == bha.BHA_OK


def test_full_prefix_validation():
    L = bha.lib()
    dm = dims()
    ws = L.bha_full_prefix_workspace_bytes(ctypes.byref(dm), 4096)
    args = lambda **kw: dict(dict(cu=A16, kvl=A16b, Q=A16c, Kc=P(0x40000), Vc=P(0x50000), cap=4096,
                                  O=P(0x60000), ws=P(0x80000), wsb=ws), **kw)

    def call(a):
        return L.bha_full_prefix_attn(ctypes.byref(dm), a["cu"], a["kvl"], a["Q"], a["Kc"], a["Vc"],
                                      a["cap"], a["O"], a["ws"], a["wsb"], NULL, NULL)
    assert call(args(kvl=NULL)) == bha.BHA_ERR_INVALID
    assert call(args(cap=-1)) == bha.BHA_ERR_INVALID
    assert call(args(Kc=MIS)) == bha.BHA_ERR_INVALID
    assert call(args(O=A16c)) == bha.BHA_ERR_INVALID
    if ws > 0:
        assert call(args(wsb=ws - 1)) == bha.BHA_ERR_INVALID


def test_kernel_variant_query():
    assert bha.kernel_variant(dims(), 1) in (0, 1)
    assert bha.kernel_variant(dims(), 4) == bha.kernel_variant(dims(), 1)  # fused: same kernels
    assert bha.kernel_variant(dims(F=3), 1) == bha.BHA_ERR_INVALID
    assert bha.kernel_variant(dims(), 9) == bha.BHA_ERR_INVALID


def test_fused_step_and_commit_validation():
    """The fused call checks what bha_hybrid_attn checks, and that no output (O, S, Z) is also
    an input or another output."""
    L = bha.lib()

    def call(dm=None, **kw):
        a = dict(cu=A16, slot=NULL, Q=A16, K=A16b, V=A16c, S=P(0x40000), Z=P(0x50000),
                 W=P(0x60000), alpha=NULL, O=P(0x70000), err=NULL)
        a.update(kw)
        return L.bha_hybrid_attn_commit(ctypes.byref(dm or dims()), a["cu"], a["slot"], a["Q"],
                                        a["K"], a["V"], a["S"], a["Z"], a["W"], a["alpha"], a["O"],
                                        a["err"], NULL)
    assert call(cu=NULL) == bha.BHA_ERR_INVALID
    assert call(S=MIS) == bha.BHA_ERR_INVALID
    assert call(O=A16) == bha.BHA_ERR_INVALID           # O aliases Q
    assert call(S=A16b) == bha.BHA_ERR_INVALID          # S aliases K
    assert call(Z=P(0x40000)) == bha.BHA_ERR_INVALID    # Z aliases S
    assert call(dims(num_slots=2)) == bha.BHA_ERR_INVALID  # identity slots need num_slots >= R
    assert call(dims(R=0)) == bha.BHA_OK                # nothing to do: no launch


def test_selftest_bounded_wait_rejects_bad_arguments_before_launching():
    L = bha.lib()
    assert L.bha_selftest_bounded_wait(1000, None, None) == -1      # no dev_err
    dummy = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    assert L.bha_selftest_bounded_wait(0, dummy, None) == -1        # limit below range
    assert L.bha_selftest_bounded_wait(5_000_000_000, dummy, None) == -1  # above range


def test_header_is_plain_c99_and_declares_every_entry_point():
    """bha.h compiles as C99 on its own (no C++ or torch types), with the argument types of
    every entry point as tests/c_header_check.c spells them."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-fsyntax-only",
                        "-I", os.path.join(root, "include"),
                        os.path.join(root, "tests", "c_header_check.c")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_teacher_splits_the_key_range_only_where_it_pays():
    """The teacher's workspace (fp32 partials of nsplit key ranges; zero when unsplit) follows
    its cost model: 64 requests x 4 KV heads already fill the GPU, so caches up to 8K tokens
    run unsplit and a 32K cache splits 4 ways; a few requests with a long cache split so that
    the key range spreads over the SMs."""
    T, Hq, d = 64 * 32, 16, 128
    per_split = T * Hq * (d + 2) * 4
    for P in (512, 2048, 8192):
        assert bha.full_prefix_workspace_bytes(64, Hq, 4, d, 32, T, P + 32) == 0
    assert bha.full_prefix_workspace_bytes(64, Hq, 4, d, 32, T, 32768 + 32) == 4 * per_split
    # 3 requests x 2 KV heads, 2000-token cache (16 tiles of 128 keys): 4 splits of 4 tiles
    assert bha.full_prefix_workspace_bytes(3, 8, 2, d, 32, 54, 2000) == 4 * 54 * 8 * (d + 2) * 4
