"""GPU parity: the CUDA path against the CPU oracle, element by element.

Small workloads (several tiles, ragged tails, odd block counts, every branch of
the routing) are compared in full: kept blocks and routing bit-exactly, outputs
within max-abs 2e-2 and relative L2 5e-3 of the float64 oracle. Intermediate
stages are compared through the debug copies of the pooled blocks, the context
scores and the sharpness.
"""
import numpy as np
import pytest

import isa_synth
from oracle import isa_oracle as O
from parity_util import compare_out, inputs, run_gpu

pytestmark = pytest.mark.gpu

W = isa_synth.Workload


def _case(name, B, H, D, L_src, L_ctx, b, a_s, a_f, dtype="bf16", sig=(0.1, 1.0), s_ctx=0.5):
    return W(name, B, H, D, L_src, L_ctx, b, a_s, a_f, sig[0], sig[1], s_ctx, dtype)


SMALL = [
    isa_synth.WORKLOADS["tiny_f32_n1024"],
    # b = 128: 16 blocks, 9 Taylor / 7 exact (an odd exact count leaves a one-tile item)
    _case("b128_h3", 1, 3, 128, 1024, 1024, 128, 0.25, 0.6),
    # b = 64: odd n_new (13 blocks -> a half-filled last K/V tile), odd n_q, half-filled query tiles
    _case("b64_ragged", 1, 2, 128, 640, 448, 64, 0.3, 0.5),
    # D = 64 in bf16
    _case("d64_b64", 1, 2, 64, 1024, 512, 64, 0.25, 0.5),
    _case("d64_b128", 1, 2, 64, 1024, 1024, 128, 0.5, 0.5),
    # several batches and heads
    _case("b2_h2", 2, 2, 128, 768, 512, 64, 0.5, 0.25),
    # every query block exact; every query block Taylor
    _case("all_exact", 1, 2, 128, 1024, 1024, 128, 0.25, 0.0),
    _case("all_taylor", 1, 2, 128, 1024, 1024, 128, 0.25, 1.0),
    # nothing kept from the context; everything kept (dense over the whole sequence at alpha_f = 0)
    _case("no_context", 1, 2, 128, 1024, 1024, 64, 0.0, 0.5),
    _case("dense_point", 1, 2, 128, 1024, 1024, 128, 1.0, 0.0),
    # long enough for several K/V tiles per item and several items per CTA
    _case("long_b128", 1, 4, 128, 4096, 4096, 128, 0.25, 0.5),
    _case("long_b64", 1, 2, 128, 4096, 2048, 64, 0.25, 0.5),
    _case("tiny_f32_ragged", 1, 2, 64, 640, 448, 64, 0.3, 0.5, dtype="f32"),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_full_parity(w):
    q, k, v = inputs(w)
    ref = O.isa_forward_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    out, sel, route = run_gpu(w, q, k, v)
    assert sel.shape == ref["sel"].shape
    np.testing.assert_array_equal(sel, ref["sel"])
    np.testing.assert_array_equal(route, ref["route"])
    compare_out(out, ref["out"])


def test_stage_intermediates():
    import torch
    import block_sparse_attention_isa_b200 as isa
    from parity_util import to_device
    w = _case("b64_ragged", 1, 2, 128, 640, 448, 64, 0.3, 0.5)
    q, k, v = inputs(w)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    pooled = isa.debug_pooled(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s)
    isa.device_status()
    for h in range(w.H):
        r = O.isa_select_route_ref(q[0, h], k[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
        np.testing.assert_allclose(pooled["qc"][0, h].cpu().numpy(), r["qc"], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(pooled["kc"][0, h].cpu().numpy(), r["kc"], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(pooled["vc"][0, h].cpu().numpy(), O.pool_blocks(v[0, h], w.b), rtol=1e-5,
                                   atol=1e-6)
        np.testing.assert_allclose(pooled["colscore"][0, h].cpu().numpy(), r["colscore"], rtol=1e-4, atol=1e-7)
        np.testing.assert_allclose(pooled["sharp"][0, h].cpu().numpy(), r["sharp"], rtol=1e-3, atol=1e-9)


def test_repeat_runs_bit_identical():
    import torch
    import block_sparse_attention_isa_b200 as isa
    from parity_util import to_device
    w = _case("b128_h3", 1, 3, 128, 1024, 1024, 128, 0.25, 0.6)
    q, k, v = inputs(w)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    a = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
    b = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
    isa.device_status()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_host_buffer_entry_matches_device_entry():
    import torch
    import block_sparse_attention_isa_b200 as isa
    from parity_util import to_device
    w = _case("b128_h3", 1, 3, 128, 1024, 1024, 128, 0.25, 0.6)
    q, k, v = inputs(w)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    dev_out = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    isa.device_status()
    hq, hk, hv = (x.cpu().pin_memory() for x in (tq, tk, tv))
    n_q, kk, _ = isa.plan(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
    sel = torch.empty((w.B, w.H, kk), dtype=torch.int32)
    route = torch.empty((w.B, w.H, n_q), dtype=torch.int32)
    host_out = isa.forward_host(hq, hk, hv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, dbg_sel=sel, dbg_route=route)
    assert torch.equal(host_out, dev_out.cpu())
    ref = O.isa_select_route_ref(q[0, 0], k[0, 0], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    np.testing.assert_array_equal(sel[0, 0].numpy(), ref["sel"])


@pytest.mark.parametrize("pinned,a_ns", [(True, 0.0), (False, 0.0), (True, 0.25)])
def test_host_buffer_pipeline_over_chunks(pinned, a_ns):
    """The host-buffer entry point runs the (batch, head) slices in chunks on three streams (copy in,
    pass, copy out). B = 2, H = 9: 18 slices in 6 chunks of 3; the result, the kept blocks and the
    routing equal the device entry point's bit for bit, with pinned and pageable host buffers."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    from parity_util import to_device
    w = _case("b128_b2_h9", 2, 9, 128, 512, 512, 128, 0.5, 0.5)
    q, k, v = isa_synth.make_inputs(w, 0)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    dev = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True, alpha_ns=a_ns)
    isa.device_status()
    hq, hk, hv = (x.cpu() for x in (tq, tk, tv))
    if pinned:
        hq, hk, hv = (x.pin_memory() for x in (hq, hk, hv))
    n_q, kk, _ = isa.plan(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s, w.alpha_f)
    sel = torch.full((w.B, w.H, kk), -1, dtype=torch.int32)
    route = torch.full((w.B, w.H, n_q), -1, dtype=torch.int32)
    host_out = isa.forward_host(hq, hk, hv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, dbg_sel=sel,
                                dbg_route=route, alpha_ns=a_ns)
    assert torch.equal(host_out, dev[0].cpu())
    assert torch.equal(sel, dev[1].cpu()) and torch.equal(route, dev[2].cpu())


def test_wait_timeout_is_reported_and_context_survives():
    import torch
    import block_sparse_attention_isa_b200 as isa
    from parity_util import to_device
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    isa.selftest_wait_timeout(ws, timeout_ms=50)
    with pytest.raises(isa.IsaError) as e:
        isa.device_status(ws)
    assert e.value.code == -6
    isa.device_status(ws)  # the word was cleared
    # the context is still usable
    w = isa_synth.WORKLOADS["tiny_f32_n1024"]
    q, k, v = inputs(w)
    ref = O.isa_forward_ref(q, k, v, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    out, sel, route = run_gpu(w, q, k, v)
    compare_out(out, ref["out"])


def test_workspace_errors_on_device():
    import torch
    import block_sparse_attention_isa_b200 as isa
    w = _case("b128_h3", 1, 3, 128, 1024, 1024, 128, 0.25, 0.6)
    x = torch.zeros((1, 3, 2048, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(isa.IsaError) as e:
        isa.forward_into(x, x, x, out, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, workspace=small)
    assert e.value.code == -4
    with pytest.raises(isa.IsaError) as e:
        isa.forward_into(x, x, x, x, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
    assert e.value.code == -1


def test_polynomial_exp2_against_cuda_exp2f():
    """The softmax's FMA-pipe 2^x stays within 1e-4 relative error of CUDA's exp2f."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    xs = np.concatenate([np.linspace(-124.0, 9.0, 200001), np.random.default_rng(0).uniform(-30, 9, 100000)])
    x = torch.tensor(xs, dtype=torch.float32, device="cuda")
    yp, yr = torch.empty_like(x), torch.empty_like(x)
    assert isa.lib().isa_selftest_exp2(x.data_ptr(), yp.data_ptr(), yr.data_ptr(), x.numel(),
                                       torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    rel = ((yp.double() - yr.double()).abs() / yr.double()).max().item()
    assert rel <= 1e-4, rel
    exact = torch.from_numpy(np.exp2(x.cpu().double().numpy()))
    assert ((yp.cpu().double() - exact).abs() / exact).max().item() <= 1e-4


def test_many_query_blocks_scoring_path():
    """n_q = 640 query blocks (above 512, where the coarse-score phase switches to 16-row items):
    kept blocks and routing bit-exact, the stage intermediates and sampled output rows close."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    from parity_util import to_device
    w = _case("many_blocks", 1, 2, 64, 20480, 20480, 64, 0.25, 0.5)
    q, k, v = inputs(w)
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    out, sel, route = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
    pooled = isa.debug_pooled(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s)
    isa.device_status()
    out = out.float().cpu().numpy()
    rng = np.random.default_rng(5)
    for h in range(w.H):
        r = O.isa_select_route_ref(q[0, h], k[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
        np.testing.assert_array_equal(sel[0, h].cpu().numpy(), r["sel"])
        np.testing.assert_array_equal(route[0, h].cpu().numpy(), np.concatenate([r["exact"], r["taylor"]]))
        np.testing.assert_allclose(pooled["colscore"][0, h].cpu().numpy(), r["colscore"], rtol=1e-4, atol=1e-7)
        np.testing.assert_allclose(pooled["sharp"][0, h].cpu().numpy(), r["sharp"], rtol=1e-3, atol=1e-9)
        rows = np.sort(rng.choice(w.N, size=192, replace=False))
        ref = O.isa_rows_ref(q[0, h], k[0, h], v[0, h], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows, sr=r)
        compare_out(out[0, h, rows], ref)


def test_maximum_block_count():
    """N / b = 2048, the largest supported block count (L_src = L_ctx = 65536, b = 64, D = 64):
    kept blocks and routing bit-exact, the stage intermediates and sampled output rows close.
    With 1024 context blocks the top-k gap rarely clears 1e-3, so this case asks 1e-4 of it
    (still about 100 times the float32 error of the context scores), 1e-3 of the routing."""
    import torch
    import block_sparse_attention_isa_b200 as isa
    from parity_util import MARGIN, to_device
    w = _case("max_blocks", 1, 1, 64, 65536, 65536, 64, 0.25, 0.5)
    for a in range(24):
        q, k, _ = isa_synth.make_slice(w, 0, 0, 0, a)
        r = O.isa_select_route_ref(q, k, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f)
        if r["topk_margin"] >= 1e-4 and r["route_margin"] >= MARGIN:
            break
    else:
        pytest.fail("no accepted attempt")
    q, k, v = isa_synth.make_inputs(w, 0, np.array([[a]], np.int64))
    tq, tk, tv = (to_device(x, w) for x in (q, k, v))
    out, sel, route = isa.forward(tq, tk, tv, w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, debug=True)
    pooled = isa.debug_pooled(w.B, w.H, w.L_src, w.L_ctx, w.D, w.b, w.alpha_s)
    isa.device_status()
    np.testing.assert_array_equal(sel[0, 0].cpu().numpy(), r["sel"])
    np.testing.assert_array_equal(route[0, 0].cpu().numpy(), np.concatenate([r["exact"], r["taylor"]]))
    np.testing.assert_allclose(pooled["colscore"][0, 0].cpu().numpy(), r["colscore"], rtol=1e-4, atol=1e-8)
    np.testing.assert_allclose(pooled["sharp"][0, 0].cpu().numpy(), r["sharp"], rtol=1e-3, atol=1e-9)
    rows = np.sort(np.random.default_rng(8).choice(w.N, size=128, replace=False))
    ref = O.isa_rows_ref(q[0, 0], k[0, 0], v[0, 0], w.L_src, w.L_ctx, w.b, w.alpha_s, w.alpha_f, rows, sr=r)
    compare_out(out.float().cpu().numpy()[0, 0, rows], ref)
