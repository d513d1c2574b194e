"""Host-side tests of the C ABI: build, symbol exports, argument checks, block counts.

No test here launches a kernel: every call either fails its host-side checks
before touching CUDA, or only computes sizes. Fake device addresses are only
ever passed together with a missing or undersized workspace, which the library
rejects before any CUDA call.
"""
import os
import re
import subprocess

import pytest

import isa_synth
import block_sparse_attention_isa_b200 as isa
from oracle import isa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "isa.h")
FAKE = 0x7F0000000000  # never dereferenced: every call below fails its checks first


@pytest.fixture(scope="module")
def L():
    from block_sparse_attention_isa_b200 import build
    build.build()
    return isa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(isa_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(isa.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", isa.lib_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (isa_[a-z0-9_]+)\b", out))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(L, name) is not None
    # nothing else leaks from the library's C++ internals
    assert all(n.startswith("isa_") for n in exported)


@pytest.mark.parametrize("name", sorted(isa_synth.all_workloads()))
def test_block_counts_match_oracle(L, name):
    w = isa_synth.all_workloads()[name]
    n_q, k, n_flat = isa.plan(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
    assert n_q == w.N // w.b
    assert k == O.kept_context_blocks(w.alpha_s, w.L_ctx // w.b)
    assert n_flat == O.taylor_block_count(w.alpha_f, n_q)


def test_headline_counts():
    assert isa.plan(1, 40, 16384, 16384, 128, 128, 0.25, 0.6) == (256, 32, 153)
    # float32 0.1 * 200 = 20.0000003 must not round up to 21
    assert isa.plan(1, 40, 25600, 25600, 128, 128, 0.1, 0.3) == (400, 20, 120)


def _fwd(L, q=FAKE, k=FAKE, v=FAKE, B=1, H=2, L_src=512, L_ctx=512, D=64, b=64, a_s=0.5, a_f=0.5, dt=0,
         out=FAKE + (1 << 32), ws=None, ws_bytes=0):
    return L.isa_forward_ex(q, k, v, B, H, L_src, L_ctx, D, b, a_s, a_f, dt, out, None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(k=None), -1), (dict(v=None), -1), (dict(out=None), -1),
    (dict(out=FAKE), -1),                      # out aliases q
    (dict(B=0), -1), (dict(H=-1), -1), (dict(L_src=0), -1), (dict(L_ctx=-64), -1),
    (dict(a_s=float("nan")), -1), (dict(a_f=1.5), -1), (dict(a_s=-0.1), -1),
    (dict(D=96), -3), (dict(b=32), -3), (dict(dt=7), -3), (dict(dt=1, D=128), -3),
    (dict(L_src=100), -4), (dict(L_ctx=96), -4),   # short last blocks are accepted: no workspace here
    (dict(L_src=65536 * 2, L_ctx=64, b=64), -3),  # N / b above 2048
    (dict(B=70000, H=1), -3),
    (dict(), -4),                                  # no workspace
    (dict(ws=FAKE + (3 << 32), ws_bytes=16), -4),  # workspace too small
])
def test_argument_errors(L, kw, code):
    assert _fwd(L, **kw) == code
    assert isa.last_error() != ""


def test_plan_and_sizes_errors(L):
    with pytest.raises(isa.IsaError) as e:
        isa.plan(1, 1, 64, 64, 80, 64, 0.5, 0.5)
    assert e.value.code == -3


def test_workspace_grows_with_size(L):
    a = isa.workspace_bytes(1, 2, 512, 512, 64, 64, 0.5, isa.ISA_F32)
    b = isa.workspace_bytes(1, 40, 16384, 16384, 128, 128, 0.25)
    assert 0 < a < b
    assert a % 256 == 0 and b % 256 == 0


def test_launch_count(L):
    assert isa.launch_count(1, 40, 16384, 16384, 128, 128, 0.25, 0.6) == 4
    assert isa.launch_count(1, 40, 16384, 16384, 128, 128, 0.0, 0.6) == 3  # nothing to gather
    assert isa.launch_count(1, 40, 100, 64, 128, 64, 0.25, 0.6) == 4  # short last blocks: same launches
    assert isa.launch_count(1, 40, 128, 64, 96, 64, 0.25, 0.6) == 0   # D = 96: invalid


def test_host_entry_rejects_before_copying(L):
    assert L.isa_forward_host(None, FAKE, FAKE, 1, 1, 64, 64, 64, 64, 0.5, 0.5, 0, FAKE + 4096, None, None) == -1
    assert L.isa_forward_host(FAKE, FAKE, FAKE, 1, 1, 64, 60, 96, 64, 0.5, 0.5, 0, FAKE + (1 << 30), None, None) == -3


# ---------------------------------------------------------------- no-sparsity ratio alpha_ns

@pytest.mark.parametrize("a_ns", [0.0, 0.01, 0.0625, 0.1, 0.125, 0.3, 0.5, 0.999, 1.0])
@pytest.mark.parametrize("name", ["tiny_f32_n1024", "bf16_n8192_b64", "bf16_n32768_b128",
                                  "bf16_n51200_b128_as0.1_af0.3_sc0.5"])
def test_no_sparse_count_matches_oracle(L, name, a_ns):
    """k_ns of the C plan equals the oracle's count and the bench's FLOP-count helper."""
    import bench
    w = isa_synth.all_workloads()[name]
    n_q, k, n_flat, k_ns = isa.plan_ns(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f, a_ns)
    assert (n_q, k, n_flat) == isa.plan(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
    n_new = w.L_src // w.b + k
    assert k_ns == O.no_sparse_block_count(a_ns, n_new) == bench.no_sparse_count(a_ns, n_new)


def test_alpha_ns_sizes_and_launches(L):
    args = (1, 40, 16384, 16384, 128, 128, 0.25)
    assert isa.plan_ns(*args, 0.6, 0.0625) == (256, 32, 153, 10)
    # the exact-block lists (int32 [BH, n_q, k_ns]) and bitmasks (uint32 [BH, n_q, ceil(n_new / 32)])
    extra = 40 * 256 * 10 * 4 + 40 * 256 * 5 * 4
    assert isa.workspace_bytes(*args, alpha_ns=0.0625) - isa.workspace_bytes(*args) == extra
    assert isa.workspace_bytes(*args, alpha_ns=0.0) == isa.workspace_bytes(*args)
    assert isa.launch_count(*args, 0.6, alpha_ns=0.0625) == 5
    assert isa.launch_count(*args, 0.6, alpha_ns=0.0) == 4
    assert isa.launch_count(*args, 0.0, alpha_ns=0.0625) == 4  # no Taylor query block: no extra launch


def _fwd_ns(L, a_ns, dt=0, D=64, ws=None, ws_bytes=0):
    return L.isa_forward_ns(FAKE, FAKE + (1 << 33), FAKE + (2 << 33), 1, 2, 512, 512, D, 64, 0.5, 0.5, a_ns, dt,
                            FAKE + (3 << 33), None, None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("a_ns,dt,code", [
    (1.5, 0, -1), (-0.1, 0, -1), (float("nan"), 0, -1),
    (0.1, 1, -3),   # float32 inputs with alpha_ns > 0
    (0.0, 1, -4),   # float32 with alpha_ns = 0 is the plain pass: fails only for the missing workspace
    (0.1, 0, -4),
])
def test_alpha_ns_argument_errors(L, a_ns, dt, code):
    assert _fwd_ns(L, a_ns, dt) == code
    assert isa.last_error() != ""


def test_bench_flops_with_alpha_ns():
    """Taylor FLOPs: each flat query row attends to n_new - k_ns pooled rows and k_ns * b keys."""
    import bench
    w = isa_synth.WORKLOADS["bf16_n32768_b128"]
    f0, f1 = bench.flops_per_call(w), bench.flops_per_call(w, 0.0625)
    assert f0 == bench.flops_per_call(w, 0.0)
    per = 4.0 * 153 * 128 * 128 * w.H  # 4 * n_flat * b * D * BH
    assert f0["taylor"] == per * 160
    assert f1["taylor"] == per * (150 + 10 * 128)
    assert f1["exact"] == f0["exact"] and f1["total"] - f0["total"] == f1["taylor"] - f0["taylor"]


def test_pass_roofline():
    """(attention FLOPs / peak + pool and gather bytes / bandwidth), as a time and over the measured one."""
    import bench
    f = {"exact": 5.0e12, "taylor": 1.0e12}
    hb = {"pool": 1.0e9, "gather": 0.5e9}
    r = bench.pass_roofline(f, hb, ms=10.0, tflops=1000.0, gbs=5000.0)
    assert abs(r["t_roof_ms"] - (6.0 + 0.3)) < 1e-9
    assert abs(r["frac"] - 0.63) < 1e-12


@pytest.mark.parametrize("L_src,L_ctx,b", [(100, 64, 64), (1000, 1100, 128), (65, 1, 64), (1, 200, 128)])
def test_ragged_block_counts(L, L_src, L_ctx, b):
    """Short last blocks: ceil(L_src / b) + ceil(L_ctx / b) blocks, k and n_flat as the ragged oracle's."""
    from oracle import isa_oracle_ragged as R
    bounds = R.block_bounds(L_src, L_ctx, b)
    n_ctx = -(-L_ctx // b)
    n_q, k, n_flat = isa.plan(1, 1, L_src, L_ctx, 64, b, 0.5, 0.5)
    assert n_q == len(bounds)
    assert k == O.kept_context_blocks(0.5, n_ctx) and n_flat == O.taylor_block_count(0.5, n_q)
    # K_new takes b rows for every block, a short one padded
    assert isa.workspace_bytes(1, 1, L_src, L_ctx, 64, b, 0.5) > 0


@pytest.mark.parametrize("which", ["q", "k", "v", "out"])
def test_misaligned_device_pointers_are_argument_errors(L, which):
    """Bulk and tensor copies need 16-byte aligned addresses: a misaligned pointer is rejected
    before any CUDA call (no workspace is given, so a missed check would return -4 instead)."""
    ptrs = dict(q=FAKE, k=FAKE + (1 << 32), v=FAKE + (2 << 32), out=FAKE + (3 << 32))
    ptrs[which] += 2  # a bf16 element off the 16-byte grid
    rc = _fwd(L, q=ptrs["q"], k=ptrs["k"], v=ptrs["v"], out=ptrs["out"])
    assert rc == -1
    assert "16-byte aligned" in isa.last_error() and which in isa.last_error()
    rc = L.isa_forward_ns(ptrs["q"], ptrs["k"], ptrs["v"], 1, 2, 512, 512, 64, 64, 0.5, 0.5, 0.25, 0,
                          ptrs["out"], None, None, None, None, 0, None)
    assert rc == -1


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_noalloc_rejects_misaligned_inputs(L, which):
    ptrs = dict(q=FAKE, k=FAKE + (1 << 32), v=FAKE + (2 << 32))
    ptrs[which] += 8
    rc = L.isa_select_context_noalloc(ptrs["q"], ptrs["k"], ptrs["v"], 1, 2, 512, 512, 64, 64, 0.5, 0,
                                      FAKE + (3 << 32), FAKE + (4 << 32), None)
    assert rc == -1
    assert "16-byte aligned" in isa.last_error()


def test_host_entry_points_take_unaligned_host_buffers(L):
    """Host buffers are copied, so their alignment is free; argument errors still come first."""
    rc = L.isa_forward_host_ns(FAKE + 2, FAKE + (1 << 32), FAKE + (2 << 32), 1, 2, 512, 512, 64, 64, 0.5, 1.5,
                               0.25, 0, FAKE + (3 << 32), None, None)
    assert rc == -1 and "alpha" in isa.last_error()


def _arr(xs):
    import ctypes
    return (ctypes.c_int32 * len(xs))(*xs)


def test_varlen_workspace_is_the_largest_element(L):
    Ls, Lc = [1000, 4096, 513], [1100, 4096, 700]
    per = [isa.workspace_bytes(1, 2, a, c, 128, 128, 0.25) for a, c in zip(Ls, Lc)]
    assert isa.varlen_workspace_bytes(2, Ls, Lc, 128, 128, 0.25) == max(per)


@pytest.mark.parametrize("Ls,Lc,code,msg", [
    ([512, 0], [512, 512], -1, "batch element 1"),       # an empty source part
    ([512, 512], [512, -3], -1, "batch element 1"),
    ([512], [512 * 4096], -3, "batch element 0"),         # block count above 2048
])
def test_varlen_rejects_bad_elements(L, Ls, Lc, code, msg):
    rc = L.isa_forward_varlen(FAKE, FAKE + (1 << 32), FAKE + (2 << 32), len(Ls), 2, _arr(Ls), _arr(Lc), 64, 64,
                              0.5, 0.5, 0, FAKE + (3 << 32), None, None, None, 0, None)
    assert rc == code
    assert msg in isa.last_error()


def test_varlen_argument_errors(L):
    # no length arrays
    assert L.isa_forward_varlen(FAKE, FAKE, FAKE, 2, 2, None, None, 64, 64, 0.5, 0.5, 0, FAKE, None, None, None, 0,
                                None) == -1
    # B = 0
    assert L.isa_forward_varlen(FAKE, FAKE, FAKE, 0, 2, _arr([1]), _arr([1]), 64, 64, 0.5, 0.5, 0, FAKE, None, None,
                                None, 0, None) == -1
    # out overlapping q over the packed batch (the second element reaches into out)
    Ls, Lc = [512, 512], [512, 512]
    assert L.isa_forward_varlen(FAKE, FAKE + (1 << 32), FAKE + (2 << 32), 2, 2, _arr(Ls), _arr(Lc), 64, 64, 0.5,
                                0.5, 0, FAKE + 2 * 1024 * 64 * 2, None, None, None, 0, None) == -1
    # misaligned v, then a missing workspace
    assert L.isa_forward_varlen(FAKE, FAKE + (1 << 32), FAKE + (2 << 32) + 4, 2, 2, _arr(Ls), _arr(Lc), 64, 64, 0.5,
                                0.5, 0, FAKE + (3 << 32), None, None, None, 0, None) == -1
    assert L.isa_forward_varlen(FAKE, FAKE + (1 << 32), FAKE + (2 << 32), 2, 2, _arr(Ls), _arr(Lc), 64, 64, 0.5,
                                0.5, 0, FAKE + (3 << 32), None, None, None, 0, None) == -4
    # more elements than supported
    big = [64] * 5000
    assert L.isa_forward_varlen(FAKE, FAKE, FAKE, 5000, 1, _arr(big), _arr(big), 64, 64, 0.5, 0.5, 0, FAKE, None,
                                None, None, 0, None) == -3


def _bwd(L, B=1, H=2, L_src=512, L_ctx=512, D=128, b=64, dt=0, ptrs=None, fws=None, fws_bytes=0, bws=None,
         bws_bytes=0):
    p = ptrs or [FAKE + (i << 32) for i in range(9)]
    return L.isa_backward(p[0], p[1], p[2], p[3], p[4], p[5], B, H, L_src, L_ctx, D, b, 0.5, 0.5, dt, p[6], p[7],
                          p[8], fws, fws_bytes, bws, bws_bytes, None)


def test_backward_workspace_bytes(L):
    # delta [BH, N] and dKc, dVc [BH, n_new, D] in float32, each part rounded up to 256 bytes
    n_new = 8 + 4  # 8 source blocks + ceil(0.5 * 8) kept
    want = 4 * 2 * 1024 + 2 * 4 * 2 * n_new * 128
    assert L.isa_backward_workspace_bytes(1, 2, 512, 512, 128, 64, 0.5, 0) == want
    assert L.isa_backward_workspace_bytes(1, 2, 512, 512, 96, 64, 0.5, 0) == 0


@pytest.mark.parametrize("kw,code,msg", [
    (dict(L_src=500), -3, "b divides"),         # a short last block
    (dict(D=64), -3, "D = 128"),
    (dict(dt=1, D=64), -3, "bfloat16"),
    (dict(), -4, "forward workspace"),           # no forward workspace
    (dict(fws=FAKE + (10 << 32), fws_bytes=1 << 30), -4, "backward workspace"),
])
def test_backward_argument_checks(L, kw, code, msg):
    assert _bwd(L, **kw) == code
    assert msg in isa.last_error()


def test_backward_pointer_checks(L):
    p = [FAKE + (i << 32) for i in range(9)]
    p[5] += 8  # dout misaligned
    assert _bwd(L, ptrs=p) == -1 and "aligned" in isa.last_error()
    p = [FAKE + (i << 32) for i in range(9)]
    p[7] = p[1] + 64  # dk inside k
    assert _bwd(L, ptrs=p) == -1 and "overlap" in isa.last_error()
    p = [FAKE + (i << 32) for i in range(9)]
    p[8] = p[6]  # dv is dq
    assert _bwd(L, ptrs=p) == -1 and "overlap" in isa.last_error()
    p = [FAKE + (i << 32) for i in range(9)]
    p[6] = p[4] + 2 * 1024 * 4  # dq right after lse (its [B, H, N] float32 extent): allowed, fails later on the workspace
    assert _bwd(L, ptrs=p) == -4
    p = [FAKE + (i << 32) for i in range(9)]
    p[3] = None
    assert _bwd(L, ptrs=p) == -1


def test_forward_train_checks(L):
    def call(lse, ws=None, ws_bytes=0):
        return L.isa_forward_train(FAKE, FAKE + (1 << 32), FAKE + (2 << 32), 1, 2, 512, 512, 128, 64, 0.5, 0.5, 0,
                                   FAKE + (3 << 32), lse, ws, ws_bytes, None)
    assert call(None) == -1 and "lse" in isa.last_error()
    assert call(FAKE + (4 << 32) + 4) == -1 and "aligned" in isa.last_error()
    assert call(FAKE + 64) == -1 and "overlap" in isa.last_error()
    assert call(FAKE + (4 << 32)) == -4  # no workspace
