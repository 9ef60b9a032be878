"""Parity of the PLE-tail backward (through the C ABI) with the CPU oracle, on a B200.

engram_ple_short_conv_backward returns dx and the fp32 gradients of the norm
scale, the convolution weights and the bias, for L = sum(dout * out) with out
the tail x + SiLU(conv(norm(x))). The kernels compute in fp32, the oracle in
fp64 from the same inputs. Bars, with o the oracle value:
  dx (fp32):           |g - o| <= 2e-5 * (1 + |o|)
  dx (bf16 / f16):     the same plus half an output ulp (2^-8 |o|, 2^-11 |o|);
  weight gradients:    |g - o| <= 1e-4 * (|o| + max |o| over the vector),
the latter for fp32 sums over up to thousands of tokens per block (a term
missed or counted twice moves a value by O(1) per token, far above the bar).
Sizes: the small branches cut across many blocks with ragged ends and the
halo rows of each block, every flag combination, kernel widths 1..4 with
dilations 1..9, empty and one-token sequences, then the page's shape
(4 x 2,560 channels, kernel 4, dilation 3) in full on 2,048 tokens and
sampled at the benchmark's 65,536 tokens.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import PLE_SHAPES, ple_inputs, row_bounds

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
ORACLE_DT = {"f32": oracle.F32, "bf16": oracle.BF16, "f16": oracle.F16}
HALF_ULP = {"f32": 0.0, "bf16": 2.0 ** -8, "f16": 2.0 ** -11}


@pytest.fixture(scope="module")
def E():
    import hashed_gram_embedding_raw_b200 as E
    torch.cuda.set_device(0)
    E.engram_get_device_error()
    return E


def dev(a, dt):
    a = np.ascontiguousarray(a)
    if dt == "f32":
        return torch.from_numpy(a.astype(np.float32)).cuda()
    return torch.from_numpy(a.view(np.int16)).view(TORCH_DT[dt]).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def grad_input(T, C, seed, dt):
    """dout ~ N(0, 1) in the gradient dtype (uint16 bits for 16-bit types)."""
    g = torch.Generator().manual_seed(9000 + seed)
    d = torch.randn((T, C), generator=g)
    if dt == "f32":
        return d.numpy()
    return d.to(TORCH_DT[dt]).view(torch.int16).numpy().view(np.uint16)


def decode(a, dt):
    """Host fp64 values of an f32 array or of 16-bit patterns (decoded on the CPU)."""
    if dt == "f32":
        return np.asarray(a, np.float64)
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
        TORCH_DT[dt]).double().numpy()


def assert_dx(got, want, dt, what=""):
    err = np.abs(got - want)
    bound = 2e-5 * (1 + np.abs(want)) + HALF_ULP[dt] * np.abs(want) * (1 + 1e-4)
    bad = err > bound
    assert not bad.any(), (f"dx {what}: {bad.sum()} of {bad.size} out of tolerance, "
                           f"max err {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}")


def assert_wgrad(got, want, name):
    err = np.abs(got - want)
    bound = 1e-4 * (np.abs(want) + np.abs(want).max())
    assert (err <= bound).all(), (name, err.max(), np.abs(want).max())


def run_both(E, x, w, nw, b, dout, cu, *, dt, gdt, wdt, group, dilation, flags=(1, 1, 1),
             eps=1e-6):
    norm, silu, res = flags
    cu_t = None if cu is None else torch.from_numpy(np.asarray(cu, np.int32)).cuda()
    dx, dnw, dw, db = E.engram_ple_short_conv_backward(
        dev(x, dt), dev(w, wdt), dev(dout, gdt), dilation=dilation, group_size=group,
        cu_seqlens=cu_t, norm_weight=None if nw is None else dev(nw, wdt),
        conv_bias=None if b is None else dev(b, wdt), eps=eps, norm=bool(norm),
        silu=bool(silu), residual=bool(res))
    torch.cuda.synchronize()
    got = (host(dx), host(dnw), host(dw), host(db))
    want = oracle.short_conv_backward(
        x, ORACLE_DT[dt], cu, w, decode(dout, gdt), dilation=dilation, group=group,
        norm_w=nw, eps=eps, bias=b, wdtype=ORACLE_DT[wdt], norm=norm, silu=silu, residual=res)
    return got, want


def check(got, want, gdt, what=""):
    assert_dx(got[0], want[0], gdt, what)
    for name, g_, w_ in zip(("dnorm_w", "dconv_w", "dbias"), got[1:], want[1:]):
        assert_wgrad(g_, w_, f"{name} {what}")


def inputs(dt, wdt, gdt, T, C, K, seed):
    x, _, _, _ = ple_inputs(T, C, K, seed, dt)
    _, nw, w, b = ple_inputs(T, C, K, seed, wdt)
    return x, nw, w, b, grad_input(T, C, seed, gdt)


@pytest.mark.parametrize("dt,gdt", [("bf16", "bf16"), ("bf16", "f32"), ("f16", "f16"),
                                    ("f32", "f32"), ("f32", "bf16")])
def test_small_branches_many_blocks(E, dt, gdt):
    s = PLE_SHAPES["ple_small"]
    T, C = s.tokens, s.channels
    x, nw, w, b, dout = inputs(dt, "f32", gdt, T, C, s.kernel, s.seed)
    cu = row_bounds(s.batch, s.seq_len)
    got, want = run_both(E, x, w, nw, b, dout, cu, dt=dt, gdt=gdt, wdt="f32", group=s.group,
                         dilation=s.dilation)
    check(got, want, gdt, f"{dt}/{gdt}")
    assert E.engram_get_device_error() == 0


@pytest.mark.parametrize("flags", [(n, si, r) for n in (0, 1) for si in (0, 1) for r in (0, 1)])
def test_flag_combinations(E, flags):
    T, C, G = 517, 512, 128
    x, nw, w, b, dout = inputs("bf16", "f32", "f32", T, C, 4, 20)
    cu = [0, 100, 100, 101, 300, 517]
    got, want = run_both(E, x, w, nw, b, dout, cu, dt="bf16", gdt="f32", wdt="f32", group=G,
                         dilation=3, flags=flags)
    check(got, want, "f32", str(flags))


@pytest.mark.parametrize("K,d", [(1, 1), (2, 1), (3, 5), (4, 1), (4, 2), (4, 3), (2, 9),
                                 (4, 9)])
def test_kernel_widths_and_dilations(E, K, d):
    T, C, G = 611, 256, 64
    x, nw, w, b, dout = inputs("bf16", "f32", "f32", T, C, K, 30 + K + d)
    cu = [0, 5, 311, 611]
    got, want = run_both(E, x, w, nw, b, dout, cu, dt="bf16", gdt="f32", wdt="f32", group=G,
                         dilation=d)
    check(got, want, "f32", f"K={K} d={d}")


@pytest.mark.parametrize("wdt", ["bf16", "f16", "f32"])
def test_weight_dtypes(E, wdt):
    T, C, G = 300, 384, 128
    x, nw, w, b, dout = inputs("bf16", wdt, "bf16", T, C, 4, 40)
    got, want = run_both(E, x, w, nw, b, dout, None, dt="bf16", gdt="bf16", wdt=wdt, group=G,
                         dilation=3)
    check(got, want, "bf16", wdt)


@pytest.mark.parametrize("G", [8, 16, 24, 648, 1288, 2552, 2560])
def test_narrow_and_widest_branches(E, G):
    # G = 8: four active threads in one warp; G = 24: a partial warp; 648: one
    # block whose last warp is partial; 1288: a cluster of 2 blocks, the
    # second narrower; 2552 and 2560 with this fp32 dout: 4 blocks of 640
    # channels (the last narrower for 2552, which is not a multiple of 16)
    C = 2 * G
    T = 97 if G < 1000 else 61
    x, nw, w, b, dout = inputs("bf16", "f32", "f32", T, C, 4, 50 + G)
    cu = [0, 1, 1, 2, 13, 40, T]
    got, want = run_both(E, x, w, nw, b, dout, cu, dt="bf16", gdt="f32", wdt="f32", group=G,
                         dilation=3)
    check(got, want, "f32", f"G={G}")


def test_f32_widest_branch(E):
    # fp32 x and dout: the smallest ring of row slots
    T, C, G = 200, 2560, 2560
    x, nw, w, b, dout = inputs("f32", "f32", "f32", T, C, 4, 55)
    got, want = run_both(E, x, w, nw, b, dout, [0, 77, 200], dt="f32", gdt="f32", wdt="f32",
                         group=G, dilation=3)
    check(got, want, "f32")


def test_no_bias_no_norm_weight(E):
    T, C, G = 200, 256, 256
    x, _, w, _, dout = inputs("f32", "f32", "f32", T, C, 4, 60)
    got, want = run_both(E, x, w, None, None, dout, None, dt="f32", gdt="f32", wdt="f32",
                         group=G, dilation=3)
    check(got, want, "f32")


def test_optional_outputs_and_empty_input(E):
    T, C, G = 64, 64, 32
    x, nw, w, b, dout = inputs("bf16", "f32", "bf16", T, C, 4, 80)
    xt, wt, gt = dev(x, "bf16"), dev(w, "f32"), dev(dout, "bf16")
    n0 = E.engram_launch_count()
    dx, dnw, dw, db = E.engram_ple_short_conv_backward(xt, wt, gt, dilation=3, group_size=G)
    torch.cuda.synchronize()
    assert E.engram_launch_count() == n0 + 2
    # the same call without the optional gradients through the raw ABI
    p = E.ConvParams(C, G, 4, 3, 1e-6, 7, E.ENGRAM_F32, 0)
    ws = torch.empty(E.engram_ple_short_conv_backward_workspace_size(C, G, 4, 3, T),
                     dtype=torch.uint8, device="cuda")
    dx2, dw2 = torch.empty_like(gt), torch.empty_like(dw)
    import ctypes
    rc = E.lib.engram_ple_short_conv_backward(
        ctypes.byref(p), xt.data_ptr(), E.ENGRAM_BF16, None, 1, T, None, wt.data_ptr(), None,
        gt.data_ptr(), E.ENGRAM_BF16, dx2.data_ptr(), None, dw2.data_ptr(), None,
        ws.data_ptr(), ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(dx2, dx) and torch.equal(dw2, dw)
    # no tokens: zero weight gradients, one launch
    empty = torch.empty((0, C), dtype=torch.bfloat16, device="cuda")
    n1 = E.engram_launch_count()
    _, dnw0, dw0, db0 = E.engram_ple_short_conv_backward(empty, wt, empty, dilation=3,
                                                         group_size=G)
    torch.cuda.synchronize()
    assert E.engram_launch_count() == n1 + 1
    assert not dnw0.any() and not dw0.any() and not db0.any()


def test_deterministic(E):
    T, C, G = 3000, 1024, 256
    x, nw, w, b, dout = inputs("bf16", "bf16", "bf16", T, C, 4, 90)
    args = (dev(x, "bf16"), dev(w, "bf16"), dev(dout, "bf16"))
    kw = dict(dilation=3, group_size=G, norm_weight=dev(nw, "bf16"), conv_bias=dev(b, "bf16"))
    r1 = E.engram_ple_short_conv_backward(*args, **kw)
    r2 = E.engram_ple_short_conv_backward(*args, **kw)
    torch.cuda.synchronize()
    for a_, b_ in zip(r1, r2):
        assert torch.equal(a_, b_)


def test_malformed_cu_seqlens_is_flagged(E):
    T, C, G = 128, 64, 32
    x, nw, w, b, dout = inputs("bf16", "f32", "bf16", T, C, 4, 95)
    E.engram_ple_short_conv_backward(dev(x, "bf16"), dev(w, "f32"), dev(dout, "bf16"),
                                     dilation=3, group_size=G,
                                     cu_seqlens=torch.tensor([0, 90, 40, T], dtype=torch.int32,
                                                             device="cuda"))
    assert E.engram_get_device_error() & E.ENGRAM_DEVERR_CU_SEQLENS


def test_rejected_arguments(E):
    x = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros_like(x)
    w = torch.zeros((64, 4), dtype=torch.float32, device="cuda")
    for kw in (dict(group_size=12), dict(group_size=48), dict(group_size=64, eps=-1.0)):
        with pytest.raises(E.EngramError):
            E.engram_ple_short_conv_backward(x, w, g, dilation=3, **kw)
    with pytest.raises(E.EngramError):            # kernel wider than 4
        E.engram_ple_short_conv_backward(x, torch.zeros((64, 5), device="cuda"), g,
                                         dilation=1, group_size=64)
    with pytest.raises(E.EngramError):            # dx overlapping dout
        E.engram_ple_short_conv_backward(x, w, g, dilation=3, group_size=64, dx=g)
    with pytest.raises(E.EngramError):            # dx overlapping x
        E.engram_ple_short_conv_backward(x, w, g, dilation=3, group_size=64, dx=x)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(E.EngramError) as e:       # workspace too small
        E.engram_ple_short_conv_backward(x, w, g, dilation=3, group_size=64, workspace=ws)
    assert e.value.status == E.ENGRAM_ENOSPC


# ------------------------------------------------------- the page's shape

def test_page_shape_in_full(E):
    s = PLE_SHAPES["ple_full"]
    T, C = 2048, s.channels
    x, nw, w, b, dout = inputs("bf16", "bf16", "bf16", T, C, s.kernel, 120)
    cu = [0, 1024, 1500, 2048]
    got, want = run_both(E, x, w, nw, b, dout, cu, dt="bf16", gdt="bf16", wdt="bf16",
                         group=s.group, dilation=s.dilation)
    check(got, want, "bf16")


def test_page_shape_benchmark_size_sampled(E):
    """The benchmark's launch: 16 x 4,096 tokens, C = 10,240 bf16. dx of sampled
    tokens (row starts and ends, block-range edges of every residue, random
    ones) against the oracle on the window of 9 tokens either side (clipped
    to the token's row), which is all that dx reads; the weight gradients of
    sampled channels against the oracle run without the norm on the oracle's
    own normalised inputs of those channels (the convolution only couples a
    channel with itself)."""
    s = PLE_SHAPES["ple_full"]
    T, C, G, K, d = s.tokens, s.channels, s.group, s.kernel, s.dilation
    halo = (K - 1) * d
    x, nw, w, b = ple_inputs(T, C, K, s.seed, "bf16")
    dout = grad_input(T, C, s.seed, "bf16")
    cu = row_bounds(s.batch, s.seq_len)
    dx, dnw, dw, db = E.engram_ple_short_conv_backward(
        dev(x, "bf16"), dev(w, "bf16"), dev(dout, "bf16"), dilation=d, group_size=G,
        cu_seqlens=torch.from_numpy(cu).cuda(), norm_weight=dev(nw, "bf16"),
        conv_bias=dev(b, "bf16"))
    torch.cuda.synchronize()
    assert E.engram_get_device_error() == 0
    gd = decode(dout, "bf16")
    rng = np.random.default_rng(8)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    chunks = max(1, sms // (s.branches * d))
    sample = {0, 1, 2, 8, 9, 10, T - 1, T - 10, 4095, 4096, 4097, 4105, 4106}
    for r in range(d):
        nr = (T - r + d - 1) // d
        for p in range(chunks + 1):
            j = nr * p // chunks
            sample |= {r + (j + e) * d for e in (-4, -3, -1, 0, 1, 3) if 0 <= r + (j + e) * d < T}
    sample |= set(int(v) for v in rng.integers(0, T, 30))
    got_dx = dx.float().cpu().numpy().astype(np.float64)
    for t in sorted(sample):
        row0 = (t // s.seq_len) * s.seq_len
        lo, hi = max(row0, t - halo), min(row0 + s.seq_len, t + halo + 1)
        want = oracle.short_conv_backward(x[lo:hi], oracle.BF16, None, w, gd[lo:hi], dilation=d,
                                          group=G, norm_w=nw, bias=b, wdtype=oracle.BF16)[0]
        assert_dx(got_dx[t], want[t - lo], "bf16", f"token {t}")
    # weight gradients of sampled channels
    chans = np.array(sorted({0, 7, 8, 2559, 2560, 5000, 10239} |
                            set(int(v) for v in rng.integers(0, C, 9))))
    n = np.empty((T, len(chans)))
    for t0 in range(0, T, 4096):
        full = oracle.grouped_rms_norm(x[t0:t0 + 4096], oracle.BF16, G, nw, oracle.BF16, 1e-6)
        n[t0:t0 + 4096] = full[:, chans]
    wc, bc = w[chans], b[chans]
    dxn, _, dwn, dbn = oracle.short_conv_backward(
        n.astype(np.float32), oracle.F32, cu, wc, gd[:, chans], dilation=d, bias=bc,
        wdtype=oracle.BF16, norm=False, residual=False)
    scale = 1.0 + decode(nw, "bf16")[chans]
    assert_wgrad(host(dw)[chans], dwn, "dconv_w")
    assert_wgrad(host(db)[chans], dbn, "dbias")
    # dn is the no-norm run's input gradient; dnorm_w = sum dn * xh = sum dn * n / (1 + w)
    assert_wgrad(host(dnw)[chans], (dxn * n).sum(0) / scale, "dnorm_w")


@pytest.mark.parametrize("T,d", [(1, 3), (5, 9), (8, 4)])
def test_fewer_tokens_than_residues(E, T, d):
    # some residues of the dilation hold no token at all
    C, G = 128, 64
    x, nw, w, b, dout = inputs("bf16", "f32", "f32", T, C, 4, 300 + T + d)
    got, want = run_both(E, x, w, nw, b, dout, None, dt="bf16", gdt="f32", wdt="f32", group=G,
                         dilation=d)
    check(got, want, "f32", f"T={T} d={d}")


def test_replays_in_a_graph(E):
    T, C, G = 4096, 5120, 2560
    x, nw, w, b, dout = inputs("bf16", "bf16", "bf16", T, C, 4, 310)
    xt, wt, gt = dev(x, "bf16"), dev(w, "bf16"), dev(dout, "bf16")
    kw = dict(dilation=3, group_size=G, norm_weight=dev(nw, "bf16"), conv_bias=dev(b, "bf16"),
              cu_seqlens=torch.tensor([0, 1000, 4096], dtype=torch.int32, device="cuda"))
    ws = torch.empty(E.engram_ple_short_conv_backward_workspace_size(C, G, 4, 3, T),
                     dtype=torch.uint8, device="cuda")
    outs = [(torch.empty_like(gt), torch.empty(C, device="cuda"),
             torch.empty((C, 4), device="cuda"), torch.empty(C, device="cuda")) for _ in range(2)]

    def call(o):
        E.engram_ple_short_conv_backward(xt, wt, gt, dx=o[0], dnorm_weight=o[1],
                                         dconv_weight=o[2], dconv_bias=o[3], workspace=ws, **kw)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call(outs[0])
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(outs[1])
    graph.replay()
    torch.cuda.synchronize()
    for a_, b_ in zip(outs[0], outs[1]):
        assert torch.equal(a_, b_)


def run_saved(E, x, w, nw, b, dout, cu, *, dt, gdt, wdt, group, dilation, K_fwd=None):
    """The forward saving every slice's inverse RMS, then the backward given
    it, against the oracle; also returns the saved values and the forward's
    outputs with and without saving."""
    cu_t = None if cu is None else torch.from_numpy(np.asarray(cu, np.int32)).cuda()
    T, C = x.shape
    xt, wt = dev(x, dt), dev(w, wdt)
    kw = dict(dilation=dilation, group_size=group, cu_seqlens=cu_t,
              norm_weight=None if nw is None else dev(nw, wdt),
              conv_bias=None if b is None else dev(b, wdt))
    inv = torch.full((T, C // group), float("nan"), device="cuda")
    out_saved = E.engram_ple_short_conv(xt, wt, inv_rms=inv, **kw)
    out_plain = E.engram_ple_short_conv(xt, wt, **kw)
    dx, dnw, dw, db = E.engram_ple_short_conv_backward(xt, wt, dev(dout, gdt), inv_rms=inv, **kw)
    torch.cuda.synchronize()
    assert E.engram_get_device_error() == 0
    got = (host(dx), host(dnw), host(dw), host(db))
    want = oracle.short_conv_backward(
        x, ORACLE_DT[dt], cu, w, decode(dout, gdt), dilation=dilation, group=group,
        norm_w=nw, bias=b, wdtype=ORACLE_DT[wdt])
    return got, want, inv.cpu().numpy().astype(np.float64), out_saved, out_plain


def oracle_inv_rms(x, dt, group):
    """Each slice's inverse RMS from the oracle's norm without a scale:
    normalised value over input at the slice's largest input."""
    n = oracle.grouped_rms_norm(x, ORACLE_DT[dt], group)
    xv = decode(x, dt)
    T, C = xv.shape
    xs = xv.reshape(T, C // group, group)
    k = np.abs(xs).argmax(axis=2)[..., None]
    return (np.take_along_axis(n.reshape(T, C // group, group), k, 2) /
            np.take_along_axis(xs, k, 2))[..., 0]


@pytest.mark.parametrize("dt,gdt,G,K", [("bf16", "bf16", 2560, 4), ("bf16", "f32", 2560, 4),
                                         ("bf16", "bf16", 1288, 4), ("f16", "f16", 520, 3),
                                         ("f32", "f32", 2560, 2), ("bf16", "bf16", 64, 1)])
def test_backward_with_the_forwards_saved_inverse_rms(E, dt, gdt, G, K):
    # clusters of 2 (bf16, 2,560 and 1,288 channels) and 4 blocks (fp32 dout
    # or x at 2,560), single blocks for narrow branches; sequence edges
    C, T = 2 * G, 301
    x, nw, w, b, dout = inputs(dt, "bf16", gdt, T, C, K, 70 + G + K)
    cu = [0, 1, 2, 40, 200, T]
    got, want, inv, out_saved, out_plain = run_saved(E, x, w, nw, b, dout, cu, dt=dt, gdt=gdt,
                                                     wdt="bf16", group=G, dilation=3)
    check(got, want, gdt, f"G={G} K={K}")
    # saving changes no output, and the saved values are the slices' inverse RMS
    assert torch.equal(out_saved, out_plain)
    ref = oracle_inv_rms(x, dt, G)
    assert np.abs(inv - ref).max() <= 1e-5 * np.abs(ref).max()


def test_saved_inverse_rms_by_the_general_forward(E):
    # kernel width 6 takes the general forward kernel; its saved values feed
    # a width-4 backward of the same x just as well (they depend on x alone)
    T, C, G = 257, 256, 128
    x, nw, w6, b, _ = inputs("bf16", "f32", "bf16", T, C, 6, 77)
    xt = dev(x, "bf16")
    inv = torch.full((T, C // G), float("nan"), device="cuda")
    E.engram_ple_short_conv(xt, dev(w6, "f32"), dilation=2, group_size=G, inv_rms=inv)
    torch.cuda.synchronize()
    ref = oracle_inv_rms(x, "bf16", G)
    got = inv.cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


def test_saved_inverse_rms_needs_the_norm(E):
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(64, 4, dtype=torch.bfloat16, device="cuda")
    inv = torch.zeros(8, 1, device="cuda")
    with pytest.raises(E.EngramError):
        E.engram_ple_short_conv(x, w, dilation=3, group_size=64, norm=False, inv_rms=inv)
    with pytest.raises(E.EngramError):
        E.engram_ple_short_conv_backward(x, w, x.clone(), dilation=3, group_size=64, norm=False,
                                         inv_rms=inv)
    with pytest.raises(ValueError):
        E.engram_ple_short_conv(x, w, dilation=3, group_size=64, inv_rms=torch.zeros(8, 2,
                                                                                     device="cuda"))
