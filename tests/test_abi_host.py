"""Host-side checks of the C ABI (no GPU needed).

The library must load without a GPU, export every entry point include/la.h
declares, and reject bad arguments synchronously before touching the device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from causal_kernelized_sequence_b200 import build, load_library
    build.build()
    return load_library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "la.h")).read()
    return sorted(set(re.findall(r"^LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", src, re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_feature_dim_and_strings(lib):
    assert lib.la_feature_dim(0, 64) == 64
    assert lib.la_feature_dim(1, 16) == 273
    assert lib.la_feature_dim(1, 0) == -1
    assert lib.la_feature_dim(7, 4) == -1
    assert lib.la_feature_dim(2, 16) == 153           # folded Taylor map
    assert lib.la_feature_dim(2, 1) == 3
    assert lib.la_status_string(0) == b"LA_OK"
    assert lib.la_status_string(4) == b"LA_ERR_TIMEOUT"
    assert lib.la_status_string(99) == b"LA_ERR_UNKNOWN"
    assert lib.la_version() >= 100


def _fwd(lib, q=0x1000, k=0x2000, v=0x3000, o=0x4000, s=None, z=None, den=None, ws=None, wsb=0,
         B=1, H=1, N=16, dqk=16, dv=16, fmap=0, dtype=0):
    P = ctypes.c_void_p
    return lib.la_forward(P(q), P(k), P(v), P(o), P(s), P(z), P(den), P(ws), wsb, B, H, N, dqk, dv,
                          fmap, dtype, None)


def test_forward_argument_errors(lib):
    assert _fwd(lib, q=None) == 1                      # null input
    assert _fwd(lib, B=0) == 1                         # non-positive size
    assert _fwd(lib, N=-3) == 1
    assert _fwd(lib, fmap=5) == 1                      # unknown feature map
    assert _fwd(lib, dtype=9) == 1                     # unknown dtype
    assert _fwd(lib, k=0x2002) == 1                    # misaligned
    assert _fwd(lib, s=0x5008) == 1                    # misaligned state
    assert _fwd(lib, fmap=1, dqk=32) == 2              # Taylor beyond d'=16: unsupported
    assert _fwd(lib, dv=256) == 2
    assert _fwd(lib, B=1 << 16, H=1 << 10, N=1 << 10) == 1   # element count overflow


def test_backward_and_decode_argument_errors(lib):
    P = ctypes.c_void_p
    good = [P(0x1000 * (i + 1)) for i in range(7)]
    args = lambda ptrs, ws=P(0x9000), wsb=1 << 20, **kw: (*ptrs, ws, wsb, kw.get("B", 1), 1, 16, 16, 16,
                                                           kw.get("fmap", 0), 0, None)
    bad = list(good); bad[3] = P(None)                 # dout missing
    assert lib.la_backward(*args(bad)) == 1
    assert lib.la_backward(*args(good, fmap=3)) == 1
    assert lib.la_backward(*args(good, B=0)) == 1
    assert lib.la_backward(*args(good, ws=P(None))) == 1            # workspace required
    assert lib.la_backward(*args(good, wsb=16 * 4)) == 1            # too small: 16 tokens x 2 fp32
    assert lib.la_backward_workspace_bytes(1, 1, 16, 16, 16, 0, 0) == 16 * 2 * 4
    # decode: q, k, v, y, s, z
    d = [P(0x1000 * (i + 1)) for i in range(6)]
    assert lib.la_decode_step(d[0], d[1], d[2], d[3], d[4], P(None), 2, 2, 16, 64, 1, 0, None) == 1
    assert lib.la_decode_step(d[0], d[1], d[2], d[3], P(0x4004), d[5], 2, 2, 16, 64, 1, 0, None) == 1
    assert lib.la_decode_step(*d, 2, 2, 17, 64, 1, 0, None) == 2


def test_feature_map_argument_errors(lib):
    P = ctypes.c_void_p
    assert lib.la_feature_map(P(None), P(0x2000), 4, 16, 1, 0, None) == 1
    assert lib.la_feature_map(P(0x1000), P(0x2000), 0, 16, 1, 0, None) == 1
    assert lib.la_feature_map(P(0x1000), P(0x2000), 4, 20, 1, 0, None) == 2


def test_workspace_bytes_invalid_is_zero(lib):
    assert lib.la_forward_workspace_bytes(0, 1, 1, 16, 16, 0, 0) == 0
    assert lib.la_backward_workspace_bytes(1, 1, 1, 16, 16, 9, 0) == 0


def test_product_path_does_not_reference_oracle():
    # The library package must never import or load the CPU oracle.
    pkg = os.path.join(ROOT, "causal_kernelized_sequence_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "la_oracle" not in txt and "import oracle" not in txt and "from oracle" not in txt, f


def test_kernel_plan_and_workspace(lib):
    import causal_kernelized_sequence_b200 as la
    # elu bf16 B=4 H=8 N=4096 D=64: 32 x 32 = 1024 chunks in 148 ranges; per
    # chunk a phi(K) tile (128 x 64 bf16) and a state snapshot (64 x 80 bf16),
    # per range two aggregates of 64 x 80 fp32.
    assert la.la_forward_workspace_bytes(4, 8, 4096, 64, 64, 0, 1) == \
        1024 * (128 * 64 * 2 + 64 * 80 * 2) + 148 * 2 * 64 * 80 * 4
    assert la.la_kernel_plan(0, 4, 8, 4096, 64, 64, 0, 1) == (2, ["fwd_split_state_kernel", "fwd_split_out_kernel"])
    # Taylor B=8 H=16: 128 heads -> no split, no workspace
    assert la.la_forward_workspace_bytes(8, 16, 2048, 16, 64, 1, 1) == 0
    assert la.la_kernel_plan(0, 8, 16, 2048, 16, 64, 1, 1)[0] == 1
    # the folded Taylor map takes the same tensor-core forward and workspace
    assert la.la_kernel_plan(0, 8, 16, 2048, 16, 64, 2, 1)[0] == 1
    assert la.la_kernel_plan(0, 1, 1, 65536, 16, 64, 2, 1) == la.la_kernel_plan(0, 1, 1, 65536, 16, 64, 1, 1)
    assert la.la_forward_workspace_bytes(1, 1, 65536, 16, 64, 2, 1) == \
        la.la_forward_workspace_bytes(1, 1, 65536, 16, 64, 1, 1) > 0
    # fp32 I/O runs on the exact CUDA-core kernel
    assert la.la_kernel_plan(0, 1, 1, 256, 32, 32, 0, 0) == (1, ["fwd_simt_kernel"])
    assert la.la_forward_workspace_bytes(1, 1, 256, 32, 32, 0, 0) == 0
    # short sequences: one range per chunk (T < 148), at most 16 ranges per head
    assert la.la_forward_workspace_bytes(1, 1, 100, 64, 64, 0, 1) == 1 * (16384 + 10240) + 1 * 2 * 5120 * 4
    assert la.la_forward_workspace_bytes(1, 2, 300, 64, 64, 0, 1) == 6 * (16384 + 10240) + 6 * 2 * 5120 * 4
    assert la.la_forward_workspace_bytes(1, 1, 16384, 64, 64, 0, 1) == 128 * (16384 + 10240) + 16 * 2 * 5120 * 4
    # elu d = 128 (and Taylor) keep the segment split: elu bf16 B=2 H=16 N=16384
    assert la.la_forward_workspace_bytes(2, 16, 16384, 128, 128, 0, 1) == 32 * 4 * 128 * 144 * 4
    # decode: vectorised kernel for dv in {32, 64, 128}
    assert la.la_kernel_plan(2, 256, 16, 1, 16, 64, 1, 0) == (1, ["decode_vec_kernel"])
    assert la.la_kernel_plan(2, 2, 2, 1, 16, 48, 0, 0) == (1, ["decode_simt_kernel"])
    assert la.la_kernel_plan(0, 0, 1, 1, 16, 16, 0, 0)[0] == -1
    # backward, elu bf16 D=128, B=2 H=16 N=16384: segment states, dq pass, R states, dk/dv pass
    n, names = la.la_kernel_plan(1, 2, 16, 16384, 128, 128, 0, 1)
    assert n == 4 and names[1] == "bwd_dq_kernel" and names[-1] == "bwd_dkdv_kernel"
    # workspace: den/dden per token + S and R increments (4 segments x 128 x 144 fp32 each)
    assert la.la_backward_workspace_bytes(2, 16, 16384, 128, 128, 0, 1) == \
        32 * 16384 * 2 * 4 + 2 * 32 * 4 * 128 * 144 * 4
    # elu d=64 and both Taylor maps (d'=16, dv=64) take the tensor-core backward too:
    # B=1 H=2 N=300 is 3 chunks, one segment each
    # (the elu increment passes run on the three-stage kernels, Taylor's on the two-stage ones)
    assert la.la_kernel_plan(1, 1, 2, 300, 64, 64, 0, 1) == \
        (4, ["bwd_sstate3_kernel", "bwd_dq_kernel", "bwd_rstate3_kernel", "bwd_dkdv_kernel"])
    assert la.la_kernel_plan(1, 1, 2, 300, 16, 64, 1, 1) == \
        (4, ["bwd_sstate_kernel", "bwd_dq_kernel", "bwd_rstate_kernel", "bwd_dkdv_kernel"])
    for fmap in (1, 2):
        assert la.la_kernel_plan(1, 8, 16, 2048, 16, 64, fmap, 1) == (2, ["bwd_dq_kernel", "bwd_dkdv_kernel"])
        # 128 heads: one segment per head, den/dden per token only
        assert la.la_backward_workspace_bytes(8, 16, 2048, 16, 64, fmap, 1) == 128 * 2048 * 2 * 4
        # 2 heads x 3 segments: plus S and R increments of 160 packed features x 80 columns
        assert la.la_backward_workspace_bytes(1, 2, 300, 16, 64, fmap, 1) == 2 * 300 * 2 * 4 + 2 * 2 * 3 * 160 * 80 * 4
    assert la.la_backward_workspace_bytes(1, 2, 300, 64, 64, 0, 1) == 2 * 300 * 2 * 4 + 2 * 2 * 3 * 64 * 80 * 4
    # the gated backward on the same shapes: plus the dL/dg suffix-sum kernel; its
    # workspace holds den, dden and c per token, and per segment the S and R
    # increments and the summed gate
    assert la.la_kernel_plan(5, 1, 2, 300, 64, 64, 0, 1) == \
        (5, ["bwd_sstate3_kernel", "bwd_dq_kernel", "bwd_rstate3_kernel", "bwd_dkdv_kernel", "bwd_dg_kernel"])
    assert la.la_kernel_plan(5, 8, 16, 2048, 16, 64, 1, 1) == (3, ["bwd_dq_kernel", "bwd_dkdv_kernel", "bwd_dg_kernel"])
    bd = la.load_library().la_backward_decay_workspace_bytes
    assert bd(1, 2, 300, 64, 64, 0, 1) == (2 * 300 * 3 + 2 * 3 * (2 * 64 * 80 + 1)) * 4
    assert bd(8, 16, 2048, 16, 64, 2, 1) == 128 * 2048 * 3 * 4
    assert bd(1, 2, 300, 32, 32, 0, 1) == 2 * 300 * 2 * 4          # CUDA-core backward: den, dden
    # fp32 and the other shapes stay on the exact CUDA-core kernel
    assert la.la_kernel_plan(1, 1, 2, 300, 32, 32, 0, 1) == (1, ["bwd_simt_kernel"])
    assert la.la_kernel_plan(1, 1, 2, 300, 64, 64, 0, 0) == (1, ["bwd_simt_kernel"])


def test_selftest_wait_limit_checked_before_launch(lib):
    lib.la_selftest_bounded_wait.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    lib.la_selftest_bounded_wait.restype = ctypes.c_int
    assert lib.la_selftest_bounded_wait(0, None) == 1
    assert lib.la_selftest_bounded_wait(2000001, None) == 1


def test_forward_from_state_argument_errors(lib):
    P = ctypes.c_void_p
    f = lib.la_forward_from_state
    f.argtypes = [P] * 10 + [ctypes.c_size_t] + [ctypes.c_int] * 7 + [P]
    f.restype = ctypes.c_int
    q, k, v, o, s_in, z_in, s_out, z_out = (0x1000 * (i + 1) for i in range(8))
    call = lambda s_in=s_in, z_in=z_in, s_out=s_out, z_out=z_out, fmap=0: \
        f(P(q), P(k), P(v), P(o), P(s_in), P(z_in), P(s_out), P(z_out), None, None, 0,
          1, 1, 16, 16, 16, fmap, 0, None)
    assert call(s_in=None) == 1                        # start state required
    assert call(z_in=None) == 1
    assert call(s_in=0x6004) == 1                      # misaligned
    assert call(s_out=s_in) == 1                       # in-place update not allowed
    assert call(z_out=z_in + 16) == 1                  # z_out overlaps z_in (16 floats)
    assert call(s_out=s_in + 16 * 16 * 4 - 16) == 1    # tail of s_in overlaps s_out
    assert call(fmap=4) == 1


def test_forward_varlen_argument_errors(lib):
    import causal_kernelized_sequence_b200 as la
    la.load_library()
    P = ctypes.c_void_p
    f = lib.la_forward_varlen
    q, k, v, o, cu = (0x1000 * (i + 1) for i in range(5))

    def call(cu=cu, nseq=2, max_len=64, T=100, s_in=None, z_in=None, ws=None, wsb=0, H=2, dqk=16, dv=64,
             fmap=1, dtype=1):
        return f(P(q), P(k), P(v), P(o), P(cu), nseq, max_len, T, P(s_in), P(z_in), None, None, None,
                 P(ws), wsb, H, dqk, dv, fmap, dtype, None)
    assert call(cu=None) == 1                          # lengths required
    assert call(cu=0x5002) == 1                        # misaligned int32 array
    assert call(T=0) == 1
    assert call(max_len=0) == 1
    assert call(nseq=0) == 1
    assert call(s_in=0x9000) == 1                      # s_in without z_in
    assert call(fmap=9) == 1
    assert call(dqk=32) == 2                           # Taylor beyond d'=16
    # one long sequence needs segment increments: the workspace is required
    need = la.la_forward_varlen_workspace_bytes(1, 1, 65536, 16, 64, 1, 1)
    assert need == la.la_forward_workspace_bytes(1, 1, 65536, 16, 64, 1, 1) > 0
    assert call(nseq=1, H=1, max_len=65536, T=65536) == 1
    assert call(nseq=1, H=1, max_len=65536, T=65536, ws=0x10000, wsb=need - 16) == 1
    # fp32 runs on the CUDA-core kernel: no workspace
    assert la.la_forward_varlen_workspace_bytes(1, 1, 65536, 16, 64, 1, 0) == 0


def test_decay_argument_errors(lib):
    P = ctypes.c_void_p
    f = lib.la_forward_decay
    f.argtypes = [P] * 11 + [ctypes.c_size_t] + [ctypes.c_int] * 7 + [P]
    f.restype = ctypes.c_int
    q, k, v, g, o = (0x1000 * (i + 1) for i in range(5))
    call = lambda g=g, s_in=None, z_in=None, N=16, fmap=0: \
        f(P(q), P(k), P(v), P(g), P(o), P(s_in), P(z_in), None, None, None, None, 0, 1, 1, N, 16, 16, fmap, 0, None)
    assert call(g=None) == 1                           # gates required
    assert call(g=0x5002) == 1                         # misaligned fp32
    assert call(s_in=0x9000) == 1                      # s_in without z_in
    assert call(N=0) == 1
    assert call(fmap=3) == 1
    d = lib.la_decode_step_decay
    d.argtypes = [P] * 7 + [ctypes.c_int] * 6 + [P]
    d.restype = ctypes.c_int
    ptr = [P(0x1000 * (i + 1)) for i in range(7)]
    assert d(ptr[0], ptr[1], ptr[2], P(None), ptr[4], ptr[5], ptr[6], 2, 2, 16, 64, 1, 0, None) == 1
    assert d(*ptr, 2, 2, 17, 64, 1, 0, None) == 2
    assert lib.la_forward_decay_workspace_bytes(2, 2, 100, 16, 64, 1, 1) == 0
    # a long gated sequence splits into segments: increments plus one summed gate each
    import causal_kernelized_sequence_b200 as la
    la.load_library()
    lib.la_forward_decay_workspace_bytes.argtypes = [ctypes.c_int] * 7
    lib.la_forward_decay_workspace_bytes.restype = ctypes.c_size_t
    P = 148
    assert lib.la_forward_decay_workspace_bytes(1, 1, 148 * 128, 16, 64, 1, 1) == P * (160 * 80 + 1) * 4
    assert lib.la_forward_decay_workspace_bytes(1, 1, 148 * 128, 16, 64, 1, 0) == 0      # fp32: CUDA cores


def test_swa_argument_errors(lib):
    P = ctypes.c_void_p
    f = lib.la_swa_forward
    f.argtypes = [P] * 5 + [ctypes.c_int] * 7 + [P]
    f.restype = ctypes.c_int
    q, k, v, o = (0x1000 * (i + 1) for i in range(4))
    call = lambda q=q, N=16, dqk=64, dv=64, w=64, dt=1, lse=None: f(P(q), P(k), P(v), P(o), P(lse), 1, 1, N, dqk, dv,
                                                                    w, dt, None)
    assert call(q=None) == 1
    assert call(w=0) == 1
    assert call(N=0) == 1
    assert call(dt=5) == 1
    assert call(q=0x1008) == 1                         # misaligned
    assert call(lse=0x9002) == 1
    assert call(w=2048) == 2                           # beyond the exact kernel's window
    assert call(dqk=256) == 2
    d = lib.la_swa_decode_step
    d.argtypes = [P] * 7 + [ctypes.c_int] * 6 + [P]
    d.restype = ctypes.c_int
    ptr = [P(0x1000 * (i + 1)) for i in range(7)]
    assert d(*ptr[:6], P(None), 1, 1, 64, 64, 64, 1, None) == 1       # positions required
    assert d(*ptr[:6], P(0x7002), 1, 1, 64, 64, 64, 1, None) == 1     # misaligned int32
    assert d(*ptr, 1, 1, 64, 64, 0, 1, None) == 1
    c = lib.la_swa_cache_fill
    c.argtypes = [P] * 4 + [ctypes.c_int] * 7 + [P]
    c.restype = ctypes.c_int
    assert c(P(None), *ptr[1:4], 1, 1, 16, 64, 64, 64, 1, None) == 1


def test_backward_decay_argument_errors(lib):
    P = ctypes.c_void_p
    f = lib.la_backward_decay
    f.argtypes = [P] * 10 + [ctypes.c_size_t] + [ctypes.c_int] * 7 + [P]
    f.restype = ctypes.c_int
    ptr = [0x1000 * (i + 1) for i in range(10)]   # q k v g dout dq dk dv dg ws
    def call(i_null=None, wsb=16 * 2 * 4, N=16):
        args = [P(None) if i == i_null else P(x) for i, x in enumerate(ptr)]
        return f(*args, wsb, 1, 1, N, 16, 16, 0, 0, None)
    for i in range(10):
        assert call(i_null=i) == 1, i              # every pointer is required
    assert call(wsb=16 * 2 * 4 - 4) == 1           # workspace too small
    assert call(N=0) == 1
    lib.la_backward_decay_workspace_bytes.argtypes = [ctypes.c_int] * 7
    lib.la_backward_decay_workspace_bytes.restype = ctypes.c_size_t
    assert lib.la_backward_decay_workspace_bytes(2, 3, 100, 16, 16, 0, 1) == 2 * 3 * 100 * 2 * 4

