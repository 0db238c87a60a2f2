"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments with the documented status before
any GPU work (these calls never reach a CUDA API, so they run without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_paro_build", os.path.join(ROOT, "rotation_w4_weight_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()                       # rebuild if a source is newer, before the library loads
    from rotation_w4_weight_b200 import _lib
    return _lib


def header_functions():
    txt = open(os.path.join(ROOT, "include", "paro.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(paro_[a-z0-9_]+)\s*\(", txt)))


def test_exports_every_header_symbol(L):
    names = header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L.lib, n), n
    assert set(names) <= set(L.EXPORTED) | set(names)
    assert L.paro_version().decode().count(".") == 2


def test_status_strings(L):
    for code in range(7):
        s = L.paro_status_string(code)
        assert s and isinstance(s, bytes)
    assert L.paro_status_string(99) == b"unknown status"


P = ctypes.c_void_p
A16 = P(0x10000)           # never dereferenced: validation fails before any use
MIS = P(0x10008)           # 8-byte aligned, not 16


def lin(L, x=A16, y=A16, M=4, K=256, N=512, qw=A16, qz=A16, sc=A16, bias=None, cs=None,
        pairs=None, theta=None, G=128, krot=0, ws=None, wsb=0):
    return L.paro_w4_linear(x, y, M, K, N, qw, qz, sc, bias, cs, pairs, theta, G, krot, ws, wsb, None)


def test_linear_argument_validation(L):
    assert lin(L, M=-1) == L.PARO_ERR_INVALID_ARG
    assert lin(L, K=0) == L.PARO_ERR_INVALID_ARG
    assert lin(L, N=12) == L.PARO_ERR_INVALID_ARG            # N % 8
    assert lin(L, N=40) == L.PARO_ERR_UNSUPPORTED            # N % 32 (valid for the packer only)
    assert lin(L, K=200) == L.PARO_ERR_INVALID_ARG           # K % G
    assert lin(L, G=3) == L.PARO_ERR_INVALID_ARG             # odd group
    # group sizes: 16, 32, 64 and 128 are implemented (checked on the GPU);
    # other valid ones are refused before any work
    assert lin(L, G=8) == L.PARO_ERR_UNSUPPORTED
    assert lin(L, K=384, G=48) == L.PARO_ERR_UNSUPPORTED
    assert lin(L, G=256) == L.PARO_ERR_UNSUPPORTED
    assert lin(L, K=256, G=-1) == L.PARO_ERR_UNSUPPORTED     # G normalised to K=256
    assert lin(L, K=64, G=-1) == L.PARO_ERR_UNSUPPORTED      # G = 64, but K must be a multiple of 128
    assert lin(L, x=None) == L.PARO_ERR_INVALID_ARG
    assert lin(L, qz=None) == L.PARO_ERR_INVALID_ARG
    assert lin(L, krot=8) == L.PARO_ERR_INVALID_ARG          # pairs/theta missing
    assert lin(L, krot=65, pairs=A16, theta=A16) == L.PARO_ERR_UNSUPPORTED
    assert lin(L, krot=-1) == L.PARO_ERR_INVALID_ARG
    assert lin(L, x=MIS) == L.PARO_ERR_ALIGNMENT
    assert lin(L, qw=MIS) == L.PARO_ERR_ALIGNMENT
    assert lin(L, cs=MIS) == L.PARO_ERR_ALIGNMENT
    assert lin(L, M=0) == L.PARO_OK                          # empty batch: no work
    need = L.paro_w4_linear_workspace_size(4, 256, 512, 128)
    assert need > 0
    # the rotated path (channel scales or krot > 0) stages X_r in the workspace
    assert lin(L, cs=A16, ws=None, wsb=0) == L.PARO_ERR_WORKSPACE
    assert lin(L, cs=A16, ws=A16, wsb=need - 1) == L.PARO_ERR_WORKSPACE
    assert lin(L, cs=A16, ws=P(0x10010), wsb=need) == L.PARO_ERR_ALIGNMENT   # needs 256 B
    assert lin(L, krot=8, pairs=A16, theta=A16, ws=None) == L.PARO_ERR_WORKSPACE


def test_workspace_size_query(L):
    f = L.paro_w4_linear_workspace_size
    assert f(4, 200, 512, 128) == 0          # rejected shape
    assert f(0, 256, 512, 128) >= 0
    # grows with M and is a multiple of 256 bytes
    for M in (1, 4, 16, 17, 2048):
        v = f(M, 4096, 4096, 128)
        assert v % 256 == 0 and v >= M * 4096 * 2
    assert f(8192, 4096, 14336, 128) >= 8192 * 4096 * 2
    # above 64 rows the rotation's R' parts (fp16 [2][K][128]) follow X_r
    assert f(65, 4096, 4096, 128) == 65 * 4096 * 2 + 2 * 4096 * 128 * 2
    assert f(64, 4096, 4096, 128) == 64 * 4096 * 2


def test_rotate_argument_validation(L):
    r = L.paro_rotate
    assert r(A16, A16, -1, 256, None, None, None, 128, 0, None) == L.PARO_ERR_INVALID_ARG
    assert r(None, A16, 4, 256, None, None, None, 128, 0, None) == L.PARO_ERR_INVALID_ARG
    assert r(A16, A16, 4, 256, None, None, None, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert r(A16, A16, 4, 256, None, A16, A16, 8, 8, None) == L.PARO_ERR_UNSUPPORTED
    assert r(A16, A16, 4, 256, None, A16, A16, 256, 8, None) == L.PARO_ERR_UNSUPPORTED
    assert r(A16, A16, 4, 250, None, A16, A16, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert r(MIS, A16, 4, 256, None, A16, A16, 128, 8, None) == L.PARO_ERR_ALIGNMENT
    assert r(A16, A16, 0, 256, None, A16, A16, 128, 8, None) == L.PARO_OK


def test_pack_argument_validation(L):
    p = L.paro_pack_awq
    assert p(A16, A16, A16, A16, 12, 256, 128, None) == L.PARO_ERR_INVALID_ARG
    assert p(A16, None, A16, A16, 16, 256, 128, None) == L.PARO_ERR_INVALID_ARG
    assert p(None, A16, A16, A16, 16, 256, 128, None) == L.PARO_ERR_INVALID_ARG
    assert p(A16, A16, P(0x10002), A16, 16, 256, 128, None) == L.PARO_ERR_ALIGNMENT
    u = L.paro_unpack_awq
    assert u(A16, A16, A16, A16, 16, 250, 128, None) == L.PARO_ERR_INVALID_ARG


def test_validate_pairs_host_helper(L):
    import synth
    lay = synth.make_layer("t", 256, 64, 3)
    import rotation_w4_weight_b200 as pb
    assert pb.validate_pairs(lay.pairs, 256, 128)
    bad = lay.pairs.copy()
    bad[2, 5] = bad[2, 6]                      # duplicate channel in a group
    assert not pb.validate_pairs(bad, 256, 128)
    bad = lay.pairs.copy()
    bad[0, 0] = 128                            # outside the group
    assert not pb.validate_pairs(bad, 256, 128)
    assert pb.validate_pairs(np.zeros((0, 256), np.int16), 256, 128, 0)


def test_quantize_argument_validation(L):
    q = L.paro_quantize_w4
    # (w, cs, pairs, theta, scales, qweight, qzeros, N, K, G, krot, stream)
    assert q(A16, None, A16, A16, A16, A16, A16, 12, 256, 128, 8, None) == L.PARO_ERR_INVALID_ARG   # N % 8
    assert q(A16, None, A16, A16, A16, A16, A16, -8, 256, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert q(A16, None, None, None, A16, A16, A16, 16, 256, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert q(None, None, A16, A16, A16, A16, A16, 16, 256, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert q(A16, None, A16, A16, None, A16, A16, 16, 256, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert q(A16, None, A16, A16, A16, A16, None, 16, 256, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert q(A16, None, A16, A16, A16, A16, A16, 16, 256, 8, 8, None) == L.PARO_ERR_UNSUPPORTED
    assert q(A16, None, A16, A16, A16, A16, A16, 16, 250, 128, 8, None) == L.PARO_ERR_INVALID_ARG
    assert q(A16, None, A16, A16, A16, A16, A16, 16, 256, 128, 65, None) == L.PARO_ERR_UNSUPPORTED
    assert q(MIS, None, A16, A16, A16, A16, A16, 16, 256, 128, 8, None) == L.PARO_ERR_ALIGNMENT
    assert q(A16, None, A16, A16, A16, P(0x10002), A16, 16, 256, 128, 8, None) == L.PARO_ERR_ALIGNMENT
    assert q(A16, None, A16, A16, A16, A16, A16, 0, 256, 128, 8, None) == L.PARO_OK   # empty: no-op


def test_group_argument_validation_and_workspace(L):
    def member(N=512, krot=8, y=A16, pairs=A16, qweight=A16):
        return L.ParoLinear(N, qweight.value, A16.value, A16.value, None, A16.value, pairs and pairs.value,
                            A16.value, krot, y and y.value)
    arr = (L.ParoLinear * 3)(member(4096), member(1024), member(1024))
    f = L.paro_w4_linear_group_workspace_size
    per = L.paro_w4_linear_workspace_size(4, 4096, 4096, 128)
    assert per > 0 and f(4, 4096, 3, arr, 128) == 3 * per
    assert f(4, 4096, 0, arr, 128) == 0 and f(4, 4096, 5, arr, 128) == 0
    g = L.paro_w4_linear_group
    assert g(A16, 4, 4096, 0, arr, 128, A16, 1 << 30, None) == L.PARO_ERR_INVALID_ARG
    assert g(A16, 4, 4096, 5, arr, 128, A16, 1 << 30, None) == L.PARO_ERR_UNSUPPORTED
    assert g(A16, 4, 4096, 3, None, 128, A16, 1 << 30, None) == L.PARO_ERR_INVALID_ARG
    bad = (L.ParoLinear * 2)(member(4096), member(1004))          # N % 8
    assert g(A16, 4, 4096, 2, bad, 128, A16, 1 << 30, None) == L.PARO_ERR_INVALID_ARG
    bad = (L.ParoLinear * 2)(member(4096), member(1024, y=None))  # no output
    assert g(A16, 4, 4096, 2, bad, 128, A16, 1 << 30, None) == L.PARO_ERR_INVALID_ARG
    bad = (L.ParoLinear * 2)(member(4096), member(1024, pairs=None))
    assert g(A16, 4, 4096, 2, bad, 128, A16, 1 << 30, None) == L.PARO_ERR_INVALID_ARG
    bad = (L.ParoLinear * 2)(member(4096), member(1024, qweight=MIS))
    assert g(A16, 4, 4096, 2, bad, 128, A16, 1 << 30, None) == L.PARO_ERR_ALIGNMENT
    assert g(MIS, 4, 4096, 3, arr, 128, A16, 1 << 30, None) == L.PARO_ERR_ALIGNMENT
    assert g(A16, 4, 4096, 3, arr, 128, None, 0, None) == L.PARO_ERR_WORKSPACE
    assert g(A16, 4, 4096, 3, arr, 128, A16, 3 * per - 1, None) == L.PARO_ERR_WORKSPACE
    assert g(A16, 4, 4096, 3, arr, 128, P(0x10010), 1 << 30, None) == L.PARO_ERR_ALIGNMENT
    assert g(A16, 0, 4096, 3, arr, 128, None, 0, None) == L.PARO_OK      # empty batch


def test_group_launch_count_query(L):
    import rotation_w4_weight_b200 as pb
    qkv = [dict(N=4096), dict(N=1024), dict(N=1024)]
    n = pb.w4_linear_group_launches(1, 4096, qkv)
    # one shared rotation launch, then one shared GEMV launch or one GEMV each
    assert n in (2, 4)
    # a member with more stages than the warp-per-row rotation takes: a
    # rotation launch per member when the GEMVs run separately
    n9 = pb.w4_linear_group_launches(1, 4096, [dict(N=4096), dict(N=1024, krot=9)])
    assert n9 in (3, 4)
    # prefill: one GEMM launch for the whole group; above 64 rows one R' build
    # and one X R' launch for all rotating members, up to 64 rows one rotation
    # launch per member
    assert pb.w4_linear_group_launches(4096, 4096, qkv) == 3
    assert pb.w4_linear_group_launches(65, 4096, qkv) == 3
    assert pb.w4_linear_group_launches(64, 4096, qkv) == 4
    assert pb.w4_linear_group_launches(17, 4096, qkv) == 4
    # prepared R' parts skip the build (one member without them still builds)
    qkv_r = [dict(m, rmat=True) for m in qkv]
    assert pb.w4_linear_group_launches(4096, 4096, qkv_r) == 2
    assert pb.w4_linear_group_launches(4096, 4096, [qkv_r[0], qkv[1]]) == 3
    assert pb.w4_linear_group_launches(4096, 4096, [dict(N=4096, rmat=True)]) == 2
    assert pb.w4_linear_group_launches(4096, 4096, [dict(N=4096)]) == 3
    assert pb.w4_linear_group_launches(1, 4096, qkv_r) in (2, 4)          # decode does not use R'
    assert pb.w4_linear_group_launches(4096, 4096, [dict(N=4096, krot=0, channel_scales=False)] * 2) == 1
    # experts sharing one rotation rotate x once: one rotation (not three) up to
    # 64 rows, and the single-rotation count on the other paths
    shared = [dict(N=1024), dict(N=1024, same_rotation_as=0), dict(N=1024, same_rotation_as=0)]
    assert pb.w4_linear_group_launches(64, 4096, shared) == 1 + 1
    assert pb.w4_linear_group_launches(4096, 4096, shared) == 2 + 1
    assert pb.w4_linear_group_launches(1, 4096, shared) in (2, 4)
    assert pb.w4_linear_group_launches(1, 4096, [dict(N=4096)]) == 2
    assert pb.w4_linear_group_launches(1, 4096, [dict(N=4096, krot=0, channel_scales=False)]) == 1
    assert pb.w4_linear_group_launches(1, 4000, qkv) == 0               # invalid K


def test_rotation_matrix_size_and_prepare_checks(L):
    assert L.paro_rotation_matrix_size(4096) == 4096 * 128 * 4
    for bad in (0, -128, 4000, 1 << 24):
        assert L.paro_rotation_matrix_size(bad) == 0, bad
    need = 4096 * 128 * 4
    prep = lambda cs=None, pr=A16, th=A16, K=4096, G=128, krot=8, dt=0, t=P(0x100000), n=need: \
        L.paro_rotation_matrix_prepare(cs, pr, th, K, G, krot, dt, t, n, None)  # noqa: E731
    assert prep(dt=2) == L.PARO_ERR_INVALID_ARG
    assert prep(K=-128) == L.PARO_ERR_INVALID_ARG
    assert prep(krot=-1) == L.PARO_ERR_INVALID_ARG
    assert prep(G=8) == L.PARO_ERR_UNSUPPORTED
    assert prep(krot=65) == L.PARO_ERR_UNSUPPORTED
    assert prep(t=None) == L.PARO_ERR_INVALID_ARG
    assert prep(pr=None) == L.PARO_ERR_INVALID_ARG
    assert prep(n=need - 1) == L.PARO_ERR_WORKSPACE
    assert prep(t=P(0x100010)) == L.PARO_ERR_ALIGNMENT
    assert prep(cs=P(0x10002)) == L.PARO_ERR_ALIGNMENT


def test_linear_rejects_misaligned_rmat(L):
    """The prepared R' pointer is checked before any launch."""
    arr = (L.ParoLinear * 1)()
    arr[0] = L.ParoLinear(512, 0x10000, 0x10000, 0x10000, None, None, None, None, 0, 0x10000, 0x100010)
    assert L.paro_w4_linear_group(A16, 4, 256, 1, arr, 128, A16, 1 << 20, None) == L.PARO_ERR_ALIGNMENT


def test_selftest_wait_limit_is_checked_on_the_host(L):
    # a zero or over-long limit is refused before any launch
    e = ctypes.c_uint64(7)
    assert L.paro_selftest_wait_timeout(0, ctypes.byref(e), None) == L.PARO_ERR_INVALID_ARG
    assert L.paro_selftest_wait_timeout(100_000_001, ctypes.byref(e), None) == L.PARO_ERR_INVALID_ARG
    assert e.value == 7


def test_dtype_entry_points_check_the_type_first(L):
    """The *_dt twins refuse a type other than fp16/bf16 before anything else,
    and otherwise check their arguments exactly as the fp16 entry points do."""
    bad = 2
    assert L.paro_rotate_dt(A16, A16, 4, 256, None, None, None, 128, 0, bad, None) == L.PARO_ERR_INVALID_ARG
    assert L.paro_quantize_w4_dt(A16, None, None, None, A16, A16, A16, 16, 256, 128, 0, bad,
                                 None) == L.PARO_ERR_INVALID_ARG
    assert L.paro_w4_linear_dt(A16, A16, 4, 256, 512, A16, A16, A16, None, None, None, None, 128, 0, -1,
                               None, 0, None) == L.PARO_ERR_INVALID_ARG
    assert L.paro_w4_linear_noalloc_dt(A16, A16, 4, 256, 512, A16, A16, A16, None, None, None, None, 128, 0, bad,
                                       None) == L.PARO_ERR_INVALID_ARG
    arr = (L.ParoLinear * 1)()
    arr[0] = L.ParoLinear(512, 0x10000, 0x10000, 0x10000, None, None, None, None, 0, 0x10000)
    assert L.paro_w4_linear_group_dt(A16, 4, 256, 1, arr, 128, bad, None, 0, None) == L.PARO_ERR_INVALID_ARG
    bf = L.PARO_DTYPE_BF16
    # with a valid type, the same statuses as the fp16 calls (no launch is reached)
    for kw, want in [(dict(M=-1), L.PARO_ERR_INVALID_ARG), (dict(N=40), L.PARO_ERR_UNSUPPORTED),
                     (dict(G=8), L.PARO_ERR_UNSUPPORTED), (dict(x=MIS), L.PARO_ERR_ALIGNMENT),
                     (dict(M=0), L.PARO_OK)]:
        a = dict(x=A16, y=A16, M=4, K=256, N=512, G=128)
        a.update(kw)
        got = L.paro_w4_linear_dt(a["x"], a["y"], a["M"], a["K"], a["N"], A16, A16, A16, None, None, None, None,
                                  a["G"], 0, bf, None, 0, None)
        assert got == want == lin(L, x=a["x"], M=a["M"], N=a["N"], G=a["G"]), kw
    assert L.paro_rotate_dt(A16, A16, 4, 256, None, A16, A16, 8, 8, bf, None) == L.PARO_ERR_UNSUPPORTED
    assert L.paro_quantize_w4_dt(A16, None, A16, A16, A16, A16, A16, 16, 256, 128, 65, bf,
                                 None) == L.PARO_ERR_UNSUPPORTED
    assert L.paro_w4_linear_noalloc_dt(A16, A16, 4, 256, 40, A16, A16, A16, None, None, None, None, 128, 0, bf,
                                       None) == L.PARO_ERR_UNSUPPORTED


def test_moe_shape_checks_and_queries(L):
    """Stacked experts: size and launch queries, and argument checks that end
    before any launch."""
    assert L.paro_w4_moe_launches(1, 4096, 4096, 64, 8, 128, 8, 1) == 3     # route gathers few rows
    assert L.paro_w4_moe_launches(4096, 4096, 4096, 64, 8, 128, 0, 0) == 3
    assert L.paro_w4_moe_launches(4096, 4096, 4096, 64, 8, 128, 8, 1) == 5   # R' build + X R' above 64 tokens
    assert L.paro_w4_moe_launches(64, 4096, 4096, 64, 8, 128, 8, 1) == 4
    assert L.paro_w4_moe_launches(1, 4096, 4096, 2048, 8, 128, 8, 1) == 0      # more experts than supported
    assert L.paro_w4_moe_launches(0, 4096, 4096, 8, 2, 128, 8, 1) == 0
    need = L.paro_w4_moe_workspace_size(16, 4096, 1024, 8, 2, 128)
    assert need >= 16 * 4096 * 2 + 32 * 4096 * 2 + 32 * (4 + 16 + 16)
    assert L.paro_w4_moe_workspace_size(16, 4096, 1024, 0, 2, 128) == 0
    assert L.paro_w4_moe_workspace_size(16, 4096, 1024, 8, 65, 128) == 0
    assert L.paro_w4_moe_workspace_size(16, 4000, 1024, 8, 2, 128) == 0
    moe = lambda x=A16, y=A16, T=16, K=4096, N=1024, E=8, k=2, idx=A16, qw=A16, qz=A16, sc=A16, cs=None, \
        krot=0, G=128, dt=0, ws=P(0x100000), n=need: L.paro_w4_moe_linear(
            x, y, T, K, N, E, k, idx, qw, qz, sc, None, cs, None, None, G, krot, dt, ws, n, None)  # noqa: E731
    assert moe(dt=2) == L.PARO_ERR_INVALID_ARG
    assert moe(T=-1) == L.PARO_ERR_INVALID_ARG
    assert moe(E=0) == L.PARO_ERR_INVALID_ARG
    assert moe(E=1025) == L.PARO_ERR_UNSUPPORTED
    assert moe(k=65) == L.PARO_ERR_UNSUPPORTED
    assert moe(G=8) == L.PARO_ERR_UNSUPPORTED
    assert moe(N=40) == L.PARO_ERR_UNSUPPORTED
    assert moe(idx=None) == L.PARO_ERR_INVALID_ARG
    assert moe(krot=8) == L.PARO_ERR_INVALID_ARG                 # pairs / theta missing
    assert moe(x=MIS) == L.PARO_ERR_ALIGNMENT
    assert moe(idx=P(0x10002)) == L.PARO_ERR_ALIGNMENT
    assert moe(ws=P(0x100010)) == L.PARO_ERR_ALIGNMENT
    assert moe(n=need - 1) == L.PARO_ERR_WORKSPACE
    assert moe(ws=None) == L.PARO_ERR_INVALID_ARG
    assert moe(T=0) == L.PARO_OK                                 # no tokens: no work


def test_rotate_rmat_checks(L):
    r = lambda x=A16, y=P(0x20000), M=4, K=256, rm=P(0x100000), dt=0: L.paro_rotate_rmat(x, y, M, K, rm, dt, None)  # noqa: E731
    assert r(dt=2) == L.PARO_ERR_INVALID_ARG
    assert r(M=-1) == L.PARO_ERR_INVALID_ARG
    assert r(K=200) == L.PARO_ERR_UNSUPPORTED
    assert r(rm=None) == L.PARO_ERR_INVALID_ARG
    assert r(y=A16) == L.PARO_ERR_INVALID_ARG          # not in place
    assert r(x=MIS) == L.PARO_ERR_ALIGNMENT
    assert r(rm=P(0x100010)) == L.PARO_ERR_ALIGNMENT
    assert r(M=0) == L.PARO_OK
