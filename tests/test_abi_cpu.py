"""C ABI checks that need no GPU: the library loads, exports every function
declared in include/moga.h, and rejects invalid arguments before touching the
device.  Fake pointer values are never dereferenced: validation fails first."""
import ctypes

import pytest

import learned_token_group_b200 as moga

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
P = 1 << 20          # a 16-byte aligned fake device address (never dereferenced)
BIG = 1 << 40


@pytest.fixture(scope="module")
def lib():
    return moga.get_lib()


def test_exports_every_declared_symbol(lib):
    names = moga.exported_names()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moga.h but not exported"


def test_version_and_status_strings(lib):
    assert lib.moga_version() >> 16 == 1
    for code, name in moga.STATUS.items():
        assert lib.moga_status_string(code).decode() == name
    assert lib.moga_status_string(99).decode() == "MOGA_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    r1 = lib.moga_route_workspace_size(1000, 16)
    r2 = lib.moga_route_workspace_size(100000, 16)
    assert 256 < r1 < r2
    a = lib.moga_group_attn_workspace_size(1000, 2, 128, 4)
    assert a >= 3 * 1000 * 2 * 128 * 2            # gathered Q, K, V
    w3 = (ctypes.c_int * 3)(3, 8, 8)
    s = lib.stga_window_attn_workspace_size(3, 8, 16, w3, 2, 128)
    assert 256 + 384 * 4 <= s < 3 * 384 * 2 * 128 * 2   # windows of up to 256 tokens: no copy, at most the window permutation
    big = (ctypes.c_int * 3)(1, 8, 16)
    frame = lib.stga_window_attn_workspace_size(3, 8, 16, big, 2, 128)
    assert frame < 3 * 384 * 2 * 128 * 2                # 128 tokens: still read in place
    big = (ctypes.c_int * 3)(3, 8, 16)
    assert lib.stga_window_attn_workspace_size(3, 8, 16, big, 2, 128) >= 3 * 384 * 2 * 128 * 2
    layer = lib.moga_layer_workspace_size(384, 2, 128, 4, 3, 8, 16, w3)
    assert layer >= max(s, lib.moga_group_attn_workspace_size(384, 2, 128, 4), lib.moga_route_workspace_size(384, 4))
    assert lib.moga_route_workspace_size(-1, 4) == 0


def _route(lib, x=P, W=P, b=None, dt=1, N=1000, d=64, M=4, out=P, ws=P, wsb=BIG):
    return lib.moga_route(x, W, b, dt, N, d, M, out, out, out, out, out, ws, wsb, None)


def test_route_validation(lib):
    assert _route(lib, x=None) == INVALID
    assert _route(lib, W=None) == INVALID
    assert _route(lib, out=None) == INVALID
    assert _route(lib, M=0) == INVALID
    assert _route(lib, M=1025) == INVALID
    assert _route(lib, dt=7) == INVALID
    assert _route(lib, N=-1) == INVALID
    assert _route(lib, d=60) == UNSUPPORTED          # bf16 rows must be 16-byte multiples
    assert _route(lib, x=P + 2) == INVALID           # misaligned
    assert _route(lib, ws=None) == INVALID
    assert _route(lib, wsb=16) == WORKSPACE


def test_sort_validation(lib):
    """moga_sort's scan keeps one shared-memory slot per group in 1024-entry
    arrays, so group counts above 1024 are refused before any launch."""
    f = lib.moga_sort
    assert f(P, 1000, 1025, P, P, P, P, BIG, None) == INVALID
    assert f(P, 1000, 2000, P, P, P, P, BIG, None) == INVALID
    assert f(P, 1000, 65536, P, P, P, P, BIG, None) == INVALID
    assert f(P, 1000, 0, P, P, P, P, BIG, None) == INVALID
    assert f(P, -1, 4, P, P, P, P, BIG, None) == INVALID
    assert f(None, 1000, 4, P, P, P, P, BIG, None) == INVALID
    assert f(P, 1000, 4, P, P, P, P, 16, None) == WORKSPACE


def _ga(lib, q=P, perm=P, N=1000, H=2, d_h=128, M=4, ws=P, wsb=BIG):
    return lib.moga_group_attn(q, q, q, perm, perm, None, N, H, d_h, M, 1.0, q, ws, wsb, None)


def test_group_attn_validation(lib):
    assert _ga(lib, q=None) == INVALID
    assert _ga(lib, perm=None) == INVALID
    assert _ga(lib, d_h=96) == UNSUPPORTED
    assert _ga(lib, H=0) == INVALID
    assert _ga(lib, M=0) == INVALID
    assert _ga(lib, N=1 << 28, H=16) == UNSUPPORTED  # N*H beyond int32 rows
    assert _ga(lib, q=P + 8) == INVALID
    assert _ga(lib, wsb=64) == WORKSPACE


def test_stga_validation(lib):
    w = (ctypes.c_int * 3)(3, 8, 8)
    bad = (ctypes.c_int * 3)(3, 0, 8)
    f = lib.stga_window_attn
    assert f(P, P, P, 3, 8, 16, None, 2, 128, 0, P, P, BIG, None) == INVALID
    assert f(P, P, P, 3, 8, 16, bad, 2, 128, 0, P, P, BIG, None) == INVALID
    assert f(P, P, P, 0, 8, 16, w, 2, 128, 0, P, P, BIG, None) == INVALID
    assert f(P, P, P, 3, 8, 16, w, 2, 128, 2, P, P, BIG, None) == INVALID
    assert f(P, P, P, 3, 8, 16, w, 2, 32, 0, P, P, BIG, None) == UNSUPPORTED
    assert f(P, P, P, 3, 8, 16, w, 2, 128, 0, P, P, 100, None) == WORKSPACE


def test_empty_input_takes_null_token_buffers(lib):
    """N = 0: the per-token pointers may be NULL; argument checks pass and
    nothing is dereferenced (a NULL workspace still fails first, so this
    runs without a GPU)."""
    f = lib.moga_layer
    args = [None, P, None, 1, None, None, None, 0, 256, 2, 128, 4, 0, 0, 0, None, None, None, None, None, P, None,
            BIG, None]
    assert f(*args) == INVALID                        # the workspace is still required
    assert lib.moga_group_attn(None, None, None, None, P, None, 0, 2, 128, 4, 1.0, None, None, BIG, None) == INVALID
    assert lib.moga_group_attn(None, None, None, None, P, None, 1, 2, 128, 4, 1.0, None, P, BIG, None) == INVALID


def test_layer_validation(lib):
    w = (ctypes.c_int * 3)(3, 8, 8)
    f = lib.moga_layer
    args = [P, P, None, 1, P, P, P, 384, 256, 2, 128, 4, 3, 8, 16, w, P, P, P, P, P, P, BIG, None]
    bad_n = list(args)
    bad_n[7] = 385                                    # N != T*Hg*Wg
    assert f(*bad_n) == INVALID
    no_ws = list(args)
    no_ws[21] = None
    assert f(*no_ws) == INVALID
    small = list(args)
    small[22] = 64
    assert f(*small) == WORKSPACE
    assert lib.moga_sync_status(None, None) == INVALID


def test_debug_inject_modes(lib):
    assert lib.moga_debug_inject(2) == INVALID
    assert lib.moga_debug_inject(-1) == INVALID
    assert lib.moga_debug_inject(0) == OK


def test_layer_ex_validation(lib):
    w = (ctypes.c_int * 3)(3, 8, 8)
    f = lib.moga_layer_ex
    args = [P, P, None, 1, P, P, P, 384, 256, 2, 128, 4, 3, 8, 16, w, 3, P, P, P, P, P, P, BIG, None]
    bad = list(args)
    bad[16] = 4                                       # unknown branch bit
    assert f(*bad) == INVALID
    bad = list(args)
    bad[15] = None                                    # STGA branch without a window
    assert f(*bad) == INVALID
    bad = list(args)
    bad[13], bad[16] = 9, 2                           # per-frame branch: grid must cover N
    assert f(*bad) == INVALID
    small = list(args)
    small[23] = 64
    assert f(*small) == WORKSPACE
    assert lib.moga_layer_ex_workspace_size(384, 2, 128, 4, 2) >= lib.moga_layer_ex_workspace_size(384, 2, 128, 4, 0)
    assert lib.moga_layer_ex_workspace_size(384, 2, 128, 4, 5) == 0


def test_route_ex_validation(lib):
    f = lib.moga_route_ex
    assert f(P, P, None, 1, 1000, 64, 4, P, P, P, P, P, P + 2, None, P, BIG, None) == INVALID  # misaligned
    assert f(P, P, None, 1, 1000, 64, 4, P, P, P, P, P, P, P, P, 256, None) == WORKSPACE
    assert lib.moga_route_ex_workspace_size(1000, 4) > lib.moga_route_workspace_size(1000, 4)


def test_wait_limit_roundtrip(lib):
    old = lib.moga_set_wait_limit_ns(123456)
    assert lib.moga_set_wait_limit_ns(old) == 123456


def test_pipe_validation(lib):
    """The host pipeline rejects bad shapes before any CUDA call, and a NULL
    handle everywhere."""
    h = ctypes.c_void_p()
    w = (ctypes.c_int * 3)(3, 8, 8)
    create = lib.moga_pipe_create
    assert create(384, 256, 2, 128, 4, 1, 3, 8, 16, w, 1, None) == INVALID          # no handle slot
    assert create(-1, 256, 2, 128, 4, 1, 0, 0, 0, None, 0, ctypes.byref(h)) == INVALID
    assert create(384, 256, 2, 96, 4, 1, 0, 0, 0, None, 0, ctypes.byref(h)) == UNSUPPORTED
    assert create(384, 256, 2, 128, 4, 7, 0, 0, 0, None, 0, ctypes.byref(h)) == INVALID  # dtype
    assert create(384, 256, 2, 128, 4, 1, 3, 8, 16, None, 1, ctypes.byref(h)) == INVALID  # window missing
    assert create(384, 256, 2, 128, 4, 1, 3, 8, 15, w, 1, ctypes.byref(h)) == INVALID     # grid != N
    assert create(384, 256, 2, 128, 4, 1, 3, 8, 16, w, 4, ctypes.byref(h)) == INVALID     # branch bits
    assert h.value is None
    assert lib.moga_pipe_submit(None, P, P, None, P, P, P, P, None, None) == INVALID
    assert lib.moga_pipe_sync(None) == INVALID
    assert lib.moga_pipe_destroy(None) == OK


def test_shot_attn_validation(lib):
    w = (ctypes.c_int * 3)(0, 15, 26)
    f = lib.stga_shot_attn
    args = [P, P, P, 20, 30, 52, w, P, 4, 2, 2, 2, 128, 1.0, 0, P, P, BIG, None]
    bad = list(args)
    bad[8] = 0                                        # no shots
    assert f(*bad) == INVALID
    bad = list(args)
    bad[8] = 21                                       # more shots than frames
    assert f(*bad) == INVALID
    bad = list(args)
    bad[9] = -1                                       # negative augmentation
    assert f(*bad) == INVALID
    bad = list(args)
    bad[7] = None                                     # shot boundaries missing
    assert f(*bad) == INVALID
    bad = list(args)
    bad[14] = 2                                       # accumulate must be 0 or 1
    assert f(*bad) == INVALID
    bad = list(args)
    bad[12] = 96
    assert f(*bad) == UNSUPPORTED
    w_bad = (ctypes.c_int * 3)(1, 0, 26)
    bad = list(args)
    bad[6] = w_bad
    assert f(*bad) == INVALID
    small = list(args)
    small[17] = 4096
    assert f(*small) == WORKSPACE
    n1 = lib.stga_shot_attn_workspace_size(20, 30, 52, w, 4, 2, 2, 2, 128)
    n2 = lib.stga_shot_attn_workspace_size(20, 30, 52, w, 8, 2, 2, 2, 128)
    assert 0 < n1 < n2
    assert lib.stga_shot_attn_workspace_size(20, 30, 52, w, 0, 2, 2, 2, 128) == 0


def test_layer_shots_validation(lib):
    w = (ctypes.c_int * 3)(0, 15, 26)
    f = lib.moga_layer_shots
    args = [P, P, None, 1, P, P, P, 9360, 256, 2, 128, 4, 6, 30, 52, w, P, 2, 2, 2, 1, P, P, P, P, P, P, BIG, None]
    bad = list(args)
    bad[20] = 2                                       # per_frame must be 0 or 1
    assert f(*bad) == INVALID
    bad = list(args)
    bad[12] = 5                                       # grid must cover N
    assert f(*bad) == INVALID
    bad = list(args)
    bad[16] = None                                    # shot boundaries missing
    assert f(*bad) == INVALID
    small = list(args)
    small[27] = 4096
    assert f(*small) == WORKSPACE
    assert lib.moga_layer_shots_workspace_size(9360, 2, 128, 4, 6, 30, 52, w, 2, 2, 2, 1) >= \
        lib.moga_layer_shots_workspace_size(9360, 2, 128, 4, 6, 30, 52, w, 2, 2, 2, 0) > 0


def test_train_validation(lib):
    w = (ctypes.c_int * 3)(3, 8, 8)
    f = lib.moga_layer_train
    Q = 0x1000010  # a second aligned fake pointer, distinct from P
    R = 0x1000020
    args = [P, P, None, 1, P, P, P, 360, 64, 2, 128, 4, 3, 10, 12, w, P, Q, R, P, P, P, P, P, P, P, BIG, None]
    bad = list(args)
    bad[17] = P                                       # o_moga must differ from out when STGA is on
    assert f(*bad) == INVALID
    bad = list(args)
    bad[18] = None                                    # o_stga missing with a window
    assert f(*bad) == INVALID
    bad = list(args)
    bad[19] = None                                    # lse_moga missing
    assert f(*bad) == INVALID
    bad = list(args)
    bad[10] = 96                                      # unsupported head dim
    assert f(*bad) == UNSUPPORTED
    small = list(args)
    small[26] = 64
    assert f(*small) == WORKSPACE
    assert lib.moga_layer_train_workspace_size(360, 2, 128, 4, 3, 10, 12, w) == \
        lib.moga_layer_workspace_size(360, 2, 128, 4, 3, 10, 12, w)


def test_backward_validation(lib):
    w = (ctypes.c_int * 3)(3, 8, 8)
    f = lib.moga_layer_backward
    args = [P, P, P, None, 1, P, P, P, 360, 64, 2, 128, 4, 3, 10, 12, w, P, P, P, P, P, P, P, P,
            P, P, None, P, P, P, P, BIG, None]
    bad = list(args)
    bad[0] = None                                     # dout missing
    assert f(*bad) == INVALID
    bad = list(args)
    bad[26] = None                                    # dW_r missing
    assert f(*bad) == INVALID
    bad = list(args)
    bad[18] = None                                    # o_stga missing with a window
    assert f(*bad) == INVALID
    bad = list(args)
    bad[13] = 4                                       # grid must cover N
    assert f(*bad) == INVALID
    bad = list(args)
    bad[12] = 0                                       # M >= 1
    assert f(*bad) == INVALID
    small = list(args)
    small[32] = 4096
    assert f(*small) == WORKSPACE
    need = lib.moga_layer_backward_workspace_size(360, 64, 2, 128, 4)
    assert need >= 4 * 360 * 2 * 128 * 2                 # head-major q, k, v and dO copies
    assert lib.moga_layer_backward_workspace_size(360, 64, 2, 96, 4) == 0


def test_train_ex_validation(lib):
    w = (ctypes.c_int * 3)(3, 8, 8)
    f = lib.moga_layer_train_ex
    Q, R, S = 0x1000010, 0x1000020, 0x1000030
    args = [P, P, None, 1, P, P, P, 360, 64, 2, 128, 4, 3, 10, 12, w, 1, P, Q, R, S, P, P, P, P, P, P, P, P, BIG,
            None]
    bad = list(args)
    bad[16] = 2                                       # per_frame must be 0 or 1
    assert f(*bad) == INVALID
    bad = list(args)
    bad[20] = None                                    # o_frame missing with per_frame
    assert f(*bad) == INVALID
    bad = list(args)
    bad[20] = R                                       # o_frame must differ from o_stga
    assert f(*bad) == INVALID
    bad = list(args)
    bad[15] = None
    bad[12] = 4                                       # per-frame alone still needs a grid covering N
    assert f(*bad) == INVALID
    assert lib.moga_layer_train_ex_workspace_size(360, 2, 128, 4, 3, 10, 12, w, 1) >= \
        lib.moga_layer_train_ex_workspace_size(360, 2, 128, 4, 3, 10, 12, w, 0) > 0
    g = lib.moga_layer_backward_ex
    gargs = [P, P, P, None, 1, P, P, P, 360, 64, 2, 128, 4, 3, 10, 12, w, 1, 0.0, P, P, P, P, P, P, P, P, P, P,
             P, P, None, P, P, P, P, BIG, None]
    bad = list(gargs)
    bad[17] = 3
    assert g(*bad) == INVALID
    bad = list(gargs)
    bad[21] = None                                    # o_frame missing with per_frame
    assert g(*bad) == INVALID
    bad = list(gargs)
    bad[18] = float("nan")                            # balance_alpha must be finite
    assert g(*bad) == INVALID
