"""GPU parity: the CUDA path (through the C ABI) against the oracle.

Codes and block scales are compared bit for bit, lr' = X_hat L1 within bf16
rounding, Y with max|Y - Y_ref| / max|Y_ref| <= 1e-2.  Shapes cover several
tiles, ragged tails, the smallest legal K and N, rank 0 (plain W4A4), GELU,
bias, LoRA attach/detach, determinism and the full-size workloads (large ones
on sampled rows: rows of the layer are independent because the activation
scale is static)."""

import numpy as np
import pytest
import torch

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from gpu_cases import Case, assert_y_close, check_act, check_y
from oracle import svdquant as S

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    status = svdq.test_bounded_wait(50_000_000)  # 50 ms
    t1.record()
    torch.cuda.synchronize()
    assert status == 1
    assert t0.elapsed_time(t1) < 5000
    # the context is still usable
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_wrong_architecture_is_refused():
    spec = WL.CFG1
    X = spec.x()
    layer = svdq.Layer(spec.w(), np.max(np.abs(X.astype(np.float32)), 0), spec.rank)
    svdq.override_device_arch(90)
    try:
        with pytest.raises(svdq.SvdqError) as e:
            layer.upload("cuda")
        assert e.value.status == svdq.ERR_UNSUPPORTED_DEVICE
    finally:
        svdq.override_device_arch(0)
    layer.upload("cuda")


def _spec_case(spec, M=None, **kw):
    return Case(spec.x(M), spec.w(), spec.rank, bias=spec.b(), **kw)


def test_cfg1_bit_exact_codes_and_output():
    case = _spec_case(WL.CFG1)
    act, Y = case.run()
    ref = check_act(case, act)
    check_y(case, Y, ref)
    case.layer.poll_status()


@pytest.mark.parametrize("M", [1, 63, 127, 129, 200, 385])
def test_ragged_rows(M):
    case = _spec_case(WL.CFG1, M=M)
    act, Y = case.run()
    check_y(case, Y, check_act(case, act))


@pytest.mark.parametrize("K,N,r", [(64, 64, 16), (128, 320, 0), (320, 192, 32), (768, 512, 48)])
def test_small_and_ragged_k_n(K, N, r):
    X = WL.make_x(130, K, seed=K + N)
    W = WL.make_w(N, K, seed=K + N)
    case = Case(X, W, r, bias=WL.make_bias(N, 5))
    act, Y = case.run()
    check_y(case, Y, check_act(case, act))


@pytest.mark.parametrize("r", [0, 16, 32, 64])
def test_ranks_including_plain_w4a4(r):
    X = WL.make_x(256, 1024, seed=r + 1)
    W = WL.make_w(768, 1024, seed=r + 1)
    case = Case(X, W, r)
    act, Y = case.run()
    check_y(case, Y, check_act(case, act))


def test_gelu_epilogue_with_bias():
    X = WL.make_x(300, 512, seed=7)
    W = WL.make_w(512, 512, seed=7)
    case = Case(X, W, 32, bias=WL.make_bias(512, 7))
    act, Y = case.run(epilogue=svdq.EPI_GELU_TANH)
    check_y(case, Y, check_act(case, act), epilogue=S.EPI_GELU_TANH)


def _same_act(case, a1, a2, M):
    """Everything kernel 1 writes (the buffers' padding is never written)."""
    for x, y in zip(case.unpack(a1, M), case.unpack(a2, M)):
        np.testing.assert_array_equal(x, y)


def test_deterministic_across_runs():
    case = _spec_case(WL.CFG2, M=512)
    act1, Y1 = case.run()
    act2, Y2 = case.run()
    _same_act(case, act1, act2, 512)
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_lora_attach_and_detach():
    spec = WL.CFG1
    case = _spec_case(spec, rank_capacity=spec.rank + 32)
    _, Y0 = case.run()
    A, B = WL.make_lora(spec.K, spec.N, 32, seed=0)
    Ad = torch.from_numpy(A.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    Bd = torch.from_numpy(B.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    case.layer.lora_swap(Ad, Bd, scale=0.75)
    assert case.layer.info().rank_total == spec.rank + 32
    S.attach_lora(case.ref, A.astype(np.float32), B.astype(np.float32), scale=0.75)
    act, Y = case.run()
    check_y(case, Y, check_act(case, act))
    case.layer.lora_swap(None)
    S.detach_lora(case.ref)
    assert case.layer.info().rank_total == spec.rank
    _, Y2 = case.run()
    assert torch.equal(Y0.view(torch.int16), Y2.view(torch.int16))


def test_activations_quantized_before_a_swap_are_refused():
    """quantize, swap, linear: the buffer's lr' columns belong to the replaced factors, so the
    linear call refuses it; quantizing again makes it usable, and the result is the adapter's."""
    spec = WL.CFG1
    case = _spec_case(spec, rank_capacity=spec.rank + 16)
    act = case.layer.quantize_act(case.Xd)
    A, B = WL.make_lora(spec.K, spec.N, 16, seed=3)
    Ad = torch.from_numpy(A.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    Bd = torch.from_numpy(B.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    case.layer.lora_swap(Ad, Bd)
    with pytest.raises(svdq.SvdqError) as e:
        case.layer.linear(act, spec.M)
    assert e.value.status == svdq.ERR_INVALID_ARGUMENT and "LoRA swap" in str(e.value)
    S.attach_lora(case.ref, A.astype(np.float32), B.astype(np.float32))
    case.layer.quantize_act(case.Xd, act)
    Y = case.layer.linear(act, spec.M)
    torch.cuda.synchronize()
    check_y(case, Y, check_act(case, act))
    case.layer.lora_swap(None)  # a detach makes the buffer stale again
    with pytest.raises(svdq.SvdqError):
        case.layer.linear(act, spec.M)


def test_swap_on_one_stream_seen_by_another_after_an_event():
    """The swap is stream ordered: a quantize + linear on a second stream that waits on an event
    recorded after the swap sees the new factors (the oracle with the adapter attached)."""
    spec = WL.CFG1
    case = _spec_case(spec, rank_capacity=spec.rank + 32)
    A, B = WL.make_lora(spec.K, spec.N, 32, seed=4)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        Ad = torch.from_numpy(A.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
        Bd = torch.from_numpy(B.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
        case.layer.lora_swap(Ad, Bd, scale=0.5, stream=s1)
        ev = torch.cuda.Event()
        ev.record(s1)
    s2.wait_event(ev)
    with torch.cuda.stream(s2):
        act = case.layer.quantize_act(case.Xd, stream=s2)
        Y = case.layer.linear(act, spec.M, stream=s2)
    s2.synchronize()
    S.attach_lora(case.ref, A.astype(np.float32), B.astype(np.float32), scale=0.5)
    check_y(case, Y, check_act(case, act))


def test_lora_over_capacity_is_refused():
    spec = WL.CFG1
    case = _spec_case(spec)
    A = torch.zeros((spec.K, 16), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((16, spec.N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svdq.SvdqError) as e:
        case.layer.lora_swap(A, B)
    assert e.value.status == svdq.ERR_UNSUPPORTED_SHAPE


# ---------------------------------------------------------- full workloads


def _rows(M, n=256, seed=0):
    g = np.random.default_rng([seed, WL.STREAM_SAMPLE])
    return np.sort(np.concatenate([[0, M - 1], g.choice(M, size=min(n, M), replace=False)]))


def test_cfg2_attention_projection_full():
    case = _spec_case(WL.CFG2)
    act, Y = case.run()
    ref = check_act(case, act)
    err = check_y(case, Y, ref)
    print(f"cfg2 max rel err {err:.3e}")
    case.layer.poll_status()


def test_cfg3_mlp_pair_sampled_rows():
    fc1 = _spec_case(WL.CFG3_FC1)
    act1, H = fc1.run(epilogue=svdq.EPI_GELU_TANH)
    rows = _rows(WL.CFG3_FC1.M, seed=3)
    ref1 = check_act(fc1, act1, rows)
    check_y(fc1, H, ref1, epilogue=S.EPI_GELU_TANH, rows=rows)
    # fc2 runs on the oracle's fc1 output (bf16), so nothing expected comes from the GPU
    h_ref = S.forward(fc1.ref, fc1.X32[rows], S.EPI_GELU_TANH)
    X2 = WL.to_bf16(h_ref)
    fc2 = Case(X2, WL.CFG3_FC2.w(), WL.CFG3_FC2.rank)
    act2, Y2 = fc2.run()
    check_y(fc2, Y2, check_act(fc2, act2))


def test_cfg4_qkv_with_lora_sampled_rows():
    spec = WL.CFG4
    case = _spec_case(spec, rank_capacity=spec.rank + spec.lora_rank)
    A, B = spec.lora()
    Ad = torch.from_numpy(A.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    Bd = torch.from_numpy(B.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    case.layer.lora_swap(Ad, Bd)
    S.attach_lora(case.ref, A.astype(np.float32), B.astype(np.float32))
    act, Y = case.run()
    rows = _rows(spec.M, seed=4)
    check_y(case, Y, check_act(case, act, rows), rows=rows)


@pytest.mark.parametrize("M,KN,r", [(256, 3072, 0), (256, 3072, 64), (4096, 3072, 16), (1024, 3072, 32)])
def test_sweep_points(M, KN, r):
    spec = WL.sweep_spec(M, KN, r)
    case = _spec_case(spec)
    act, Y = case.run()
    rows = _rows(M, seed=5)
    check_y(case, Y, check_act(case, act, rows), rows=rows)


def test_two_calls_share_nothing_between_layers():
    a = _spec_case(WL.CFG1)
    b = Case(WL.make_x(64, 256, seed=9), WL.make_w(256, 256, seed=9), 16)
    act_a, Ya = a.run()
    act_b, Yb = b.run()
    act_a2, Ya2 = a.run()
    assert torch.equal(Ya.view(torch.int16), Ya2.view(torch.int16))
    check_y(b, Yb, check_act(b, act_b))
    _same_act(a, act_a, act_a2, 64)


def test_clone_on_another_buffer_gives_identical_output():
    spec = WL.CFG1
    case = _spec_case(spec, rank_capacity=spec.rank + 16)
    _, Y0 = case.run()
    A, B = WL.make_lora(spec.K, spec.N, 16, seed=1)
    Ad = torch.from_numpy(A.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    Bd = torch.from_numpy(B.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    case.layer.lora_swap(Ad, Bd)  # the clone must not inherit the adapter
    twin = case.layer.clone(device="cuda")
    assert twin.info().rank_total == spec.rank
    act = twin.quantize_act(case.Xd)
    Y1 = twin.linear(act, spec.M)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))
    twin.poll_status()


def test_largest_sweep_point_on_sampled_outputs():
    """M = 16384 tokens, K = N = 12288, rank 64: the largest sweep point, run whole on
    the GPU and checked on 128 sampled rows x 64 sampled output features.

    The low-rank factors are seeded N(0, 0.05) bf16 values given to both sides
    (a LAPACK SVD of this size does not fit the test's time); the oracle
    prepares only the sampled output features (lambda and g_w still come from
    the whole weight).  Codes and scales of the sampled rows are compared bit
    for bit, Y within the layer tolerance."""
    from oracle import formats as F
    from gpu_cases import LR_TOL

    spec = WL.sweep_spec(16384, 12288, 64)
    X, W = spec.x(), spec.w()
    X32 = X.astype(np.float32)
    amax = np.max(np.abs(X32), axis=0)
    g = np.random.default_rng([spec.seed, WL.STREAM_SAMPLE, 2])
    l1 = S.bf16_from_f64(g.normal(0.0, 0.05, (spec.K, spec.rank)))
    l2 = S.bf16_from_f64(g.normal(0.0, 0.05, (spec.rank, spec.N)))
    cols = np.sort(np.concatenate([[0, spec.N - 1], g.choice(spec.N, size=62, replace=False)]))
    rows = _rows(spec.M, n=126, seed=6)
    ref = S.prepare(W.astype(np.float32), amax, spec.rank, factors=(l1, l2), out_rows=cols)
    layer = svdq.Layer(W, amax, spec.rank, factors=(F.bf16_bits(l1.astype(np.float32)),
                                                     F.bf16_bits(l2.astype(np.float32))), device="cuda")
    Xd = torch.from_numpy(X.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    act = layer.quantize_act(Xd)
    Y = layer.linear(act, spec.M)
    torch.cuda.synchronize()
    layer.poll_status()
    codes, scales, lr = layer.act_unpack(act.cpu().numpy(), spec.M)
    ref_act = S.quantize_act(ref, X32[rows])
    np.testing.assert_array_equal(codes[rows], F.pack_e2m1(ref_act.codes))
    np.testing.assert_array_equal(scales[rows], ref_act.scales)
    lr_gpu = F.bf16_from_bits(lr[rows]).astype(np.float64) * ref.alpha
    assert np.max(np.abs(lr_gpu - ref_act.lr)) <= LR_TOL * np.max(np.abs(ref_act.lr))
    y = Y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    assert_y_close(y, S.linear(ref, ref_act))


@pytest.mark.parametrize("M,K,N,r", [(300, 1024, 512, 128), (200, 2048, 256, 256)])
def test_large_ranks_up_to_the_capacity_limit(M, K, N, r):
    # rank 256 is the capacity limit: kernel 1 reduces its float partials by
    # pulling them from the cluster (the push buffer no longer fits beside the
    # stages) and kernel 2 folds four 64-rank chunks
    case = Case(WL.make_x(M, K, seed=r), WL.make_w(N, K, seed=r), r, bias=WL.make_bias(N, seed=r))
    act, Y = case.run()
    err = check_y(case, Y, check_act(case, act))
    print(f"M{M} K{K} N{N} r{r}: max rel err {err:.3e}")
    case.layer.poll_status()


def test_lora_filling_the_rank_capacity():
    # rank 240 + a 16-rank adapter = 256, the largest total the layer takes
    M, K, N = 130, 512, 320
    case = Case(WL.make_x(M, K, seed=33), WL.make_w(N, K, seed=33), 240, rank_capacity=256)
    A, B = WL.make_lora(K, N, 16, seed=33)
    Ad = torch.from_numpy(A.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    Bd = torch.from_numpy(B.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    case.layer.lora_swap(Ad, Bd)
    S.attach_lora(case.ref, A.astype(np.float32), B.astype(np.float32))
    act, Y = case.run()
    check_y(case, Y, check_act(case, act))
    assert case.layer.info().rank_total == 256
    case.layer.poll_status()


def test_graph_replay_of_the_bench_step_matches_direct_launches():
    """The bench times kernel 1 + kernel 2 captured in one CUDA graph (linked by
    programmatic dependent launch) over rotating buffer sets.  Replaying such a
    graph gives the direct launches' output bit for bit, on every set."""
    import bench

    M = 1024
    case = _spec_case(WL.CFG2, M=M)
    act_ref, Y_ref = case.run()
    check_y(case, Y_ref, check_act(case, act_ref))
    layers = [case.layer, case.layer.clone(device="cuda")]
    Xs = [case.Xd, case.Xd.clone()]
    acts = [L.new_act_buffer(M) for L in layers]
    Ys = [torch.empty((M, WL.CFG2.N), dtype=torch.bfloat16, device="cuda") for _ in layers]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(2):  # eager warm-up, as the bench does before capturing
            layers[i].quantize_act(Xs[i], acts[i])
            layers[i].linear(acts[i], M, out=Ys[i])
        stream.synchronize()
    fns = []
    for i in range(2):
        fns.append(lambda i=i: layers[i].quantize_act(Xs[i], acts[i]))
        fns.append(lambda i=i: layers[i].linear(acts[i], M, out=Ys[i]))
    graph = bench._capture(fns, stream)
    for Y in Ys:
        Y.zero_()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(3):
            graph.replay()
    torch.cuda.synchronize()
    for Y in Ys:
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    for L in layers:
        L.poll_status()
    del graph


def test_layer_imported_from_a_blob_gives_the_same_output():
    """A checkpoint round trip: serialize, import, upload; the imported layer's activation buffer
    and Y are bit-identical to the original's, and within tolerance of the oracle."""
    spec = WL.CFG1
    case = _spec_case(spec)
    act0, Y0 = case.run()
    b = svdq.Layer.from_blob(case.layer.serialize(), device="cuda")
    act1 = b.quantize_act(case.Xd)
    Y1 = b.linear(act1, spec.M)
    torch.cuda.synchronize()
    _same_act(case, act0, act1, spec.M)
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))
    check_y(case, Y1, check_act(case, act1))
    b.poll_status()
