"""Parity of the PLE tail kernels (through the C ABI) with the CPU oracle, on a B200.

engram_ple_short_conv = x + SiLU(causal depthwise conv(grouped RMS norm(x)))
with each step switchable, and engram_grouped_rms_norm. The kernels compute in
fp32 and round once; the oracle computes in fp64. Bar, per element, with o
the oracle value:
  fp32 output:       |g - o| <= 2e-5 * (1 + |o|)
  bf16 / f16 output: the same plus half an output ulp (2^-8 |o| for bf16,
                     2^-11 |o| for f16) for the final rounding.
The 2e-5 bound covers the fp32 sum of squares over a 2,560-wide branch, the
approximate rsqrt / exp / reciprocal and four fused multiply-adds on O(1)
inputs. Sizes: branches cut across many blocks with ragged ends and halo rows,
every flag combination, kernel widths 1..8, empty and one-token sequences,
then the page's shape (4 x 2,560 channels, kernel 4, dilation 3) in full on
2,048 tokens and sampled at the benchmark's 65,536 tokens.
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
    """Device tensor of dtype dt from a host array (uint16 bit patterns for 16-bit)."""
    a = np.ascontiguousarray(a)
    if dt == "f32":
        return torch.from_numpy(a.astype(np.float32)).cuda()
    return torch.from_numpy(a.view(np.int16)).view(TORCH_DT[dt]).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_close(got, want, out_dt, what=""):
    err = np.abs(got - want)
    bound = 2e-5 * (1 + np.abs(want)) + HALF_ULP[out_dt] * np.abs(want) * (1 + 1e-4)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} out of tolerance, "
                           f"max err {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}")


def run_conv(E, x, w, nw, b, cu, *, dt, wdt, out_dt, group, dilation, flags=(1, 1, 1),
             eps=1e-6):
    norm, silu, res = flags
    out = E.engram_ple_short_conv(
        dev(x, dt), dev(w, wdt), dilation=dilation, group_size=group,
        cu_seqlens=None if cu is None else torch.from_numpy(np.asarray(cu, np.int32)).cuda(),
        norm_weight=None if nw is None else dev(nw, wdt),
        conv_bias=None if b is None else dev(b, wdt), eps=eps, norm=bool(norm),
        silu=bool(silu), residual=bool(res), out_dtype=TORCH_DT[out_dt])
    torch.cuda.synchronize()
    return host(out)


def oracle_conv(x, w, nw, b, cu, *, dt, wdt, group, dilation, flags=(1, 1, 1), eps=1e-6):
    norm, silu, res = flags
    return oracle.short_conv(x, ORACLE_DT[dt], cu, w, dilation=dilation, group=group,
                             norm_w=nw, eps=eps, bias=b, wdtype=ORACLE_DT[wdt], norm=norm,
                             silu=silu, residual=res)


def small_inputs(dt, wdt, T, C, K, seed):
    x, _, _, _ = ple_inputs(T, C, K, seed, dt)
    _, nw, w, b = ple_inputs(T, C, K, seed, wdt)
    return x, nw, w, b


# ------------------------------------------------------------ convolution

@pytest.mark.parametrize("dt,out_dt", [("bf16", "bf16"), ("bf16", "f32"), ("f16", "f16"),
                                       ("f16", "f32"), ("f32", "f32")])
def test_small_branches_many_blocks(E, dt, out_dt):
    s = PLE_SHAPES["ple_small"]
    T, C = s.tokens, s.channels
    x, nw, w, b = small_inputs(dt, "f32", T, C, s.kernel, s.seed)
    cu = row_bounds(s.batch, s.seq_len)
    got = run_conv(E, x, w, nw, b, cu, dt=dt, wdt="f32", out_dt=out_dt, group=s.group,
                   dilation=s.dilation)
    want = oracle_conv(x, w, nw, b, cu, dt=dt, wdt="f32", group=s.group, dilation=s.dilation)
    assert_close(got, want, out_dt)
    assert E.engram_get_device_error() == 0


@pytest.mark.parametrize("flags", [(n, si, r) for n in (0, 1) for si in (0, 1) for r in (0, 1)])
def test_flag_combinations(E, flags):
    T, C, G = 517, 512, 128
    x, nw, w, b = small_inputs("bf16", "f32", T, C, 4, 20)
    cu = [0, 100, 100, 101, 300, 517]
    got = run_conv(E, x, w, nw, b, cu, dt="bf16", wdt="f32", out_dt="f32", group=G,
                   dilation=3, flags=flags)
    want = oracle_conv(x, w, nw, b, cu, dt="bf16", wdt="f32", group=G, dilation=3, flags=flags)
    assert_close(got, want, "f32", str(flags))


@pytest.mark.parametrize("K,d", [(1, 1), (2, 1), (3, 5), (4, 1), (4, 3), (5, 7), (8, 2),
                                 (8, 9), (4, 257)])
def test_kernel_widths_and_dilations(E, K, d):
    T, C, G = 611, 256, 64
    x, nw, w, b = small_inputs("bf16", "f32", T, C, K, 30 + K + d)
    cu = [0, 5, 311, 611]
    got = run_conv(E, x, w, nw, b, cu, dt="bf16", wdt="f32", out_dt="f32", group=G, dilation=d)
    want = oracle_conv(x, w, nw, b, cu, dt="bf16", wdt="f32", group=G, dilation=d)
    assert_close(got, want, "f32", f"K={K} d={d}")


@pytest.mark.parametrize("wdt", ["bf16", "f16", "f32"])
def test_weight_dtypes(E, wdt):
    T, C, G = 300, 384, 128
    x, nw, w, b = small_inputs("bf16", wdt, T, C, 4, 40)
    got = run_conv(E, x, w, nw, b, None, dt="bf16", wdt=wdt, out_dt="f32", group=G, dilation=3)
    want = oracle_conv(x, w, nw, b, None, dt="bf16", wdt=wdt, group=G, dilation=3)
    assert_close(got, want, "f32", wdt)


@pytest.mark.parametrize("G", [8, 16, 24, 3376])
def test_narrow_and_widest_branches(E, G):
    # G = 8: one active thread per block; G = 24: a partial warp; G = 3376: a
    # branch wider than 2,560 (the chunked kernel, 8 channels per thread)
    C = 2 * G if G < 1000 else G
    T = 97 if G < 1000 else 61
    x, nw, w, b = small_inputs("bf16", "f32", T, C, 4, 50 + G)
    cu = [0, 1, 1, 2, 13, 40, T]
    got = run_conv(E, x, w, nw, b, cu, dt="bf16", wdt="f32", out_dt="f32", group=G, dilation=3)
    want = oracle_conv(x, w, nw, b, cu, dt="bf16", wdt="f32", group=G, dilation=3)
    assert_close(got, want, "f32", f"G={G}")


def test_no_bias_no_norm_weight(E):
    T, C, G = 200, 256, 256
    x, _, w, _ = small_inputs("f32", "f32", T, C, 4, 60)
    got = run_conv(E, x, w, None, None, None, dt="f32", wdt="f32", out_dt="f32", group=G,
                   dilation=3)
    want = oracle_conv(x, w, None, None, None, dt="f32", wdt="f32", group=G, dilation=3)
    assert_close(got, want, "f32")


def test_zero_start_convolution_returns_input_bits(E):
    # init_weights' zero-start convolution: the tail is then the residual alone
    T, C, G = 333, 1024, 256
    x, nw, _, _ = small_inputs("bf16", "bf16", T, C, 4, 70)
    w = np.zeros((C, 4), np.uint16)
    xt = dev(x, "bf16")
    out = E.engram_ple_short_conv(xt, dev(w, "bf16"), dilation=3, group_size=G,
                                  norm_weight=dev(nw, "bf16"))
    assert torch.equal(out.view(torch.int16), xt.view(torch.int16))


def test_launch_count_and_empty_input(E):
    T, C, G = 64, 64, 32
    x, nw, w, b = small_inputs("bf16", "f32", T, C, 4, 80)
    n0 = E.engram_launch_count()
    run_conv(E, x, w, nw, b, None, dt="bf16", wdt="f32", out_dt="bf16", group=G, dilation=3)
    assert E.engram_launch_count() == n0 + 1
    empty = torch.empty((0, C), dtype=torch.bfloat16, device="cuda")
    E.engram_ple_short_conv(empty, dev(w, "f32"), dilation=3, group_size=G)
    assert E.engram_launch_count() == n0 + 1


def test_malformed_cu_seqlens_is_flagged(E):
    T, C, G = 128, 64, 32
    x, nw, w, b = small_inputs("bf16", "f32", T, C, 4, 90)
    run_conv(E, x, w, nw, b, [0, 90, 40, T], dt="bf16", wdt="f32", out_dt="bf16", group=G,
             dilation=3)
    assert E.engram_get_device_error() & E.ENGRAM_DEVERR_CU_SEQLENS


def test_rejected_arguments(E):
    x = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((64, 4), dtype=torch.float32, device="cuda")
    for kw in (dict(group_size=12), dict(group_size=48), dict(group_size=64, eps=-1.0)):
        with pytest.raises(E.EngramError):
            E.engram_ple_short_conv(x, w, dilation=3, **kw)
    with pytest.raises(E.EngramError):            # kernel wider than 8
        E.engram_ple_short_conv(x, torch.zeros((64, 9), device="cuda"), dilation=1,
                                group_size=64)
    with pytest.raises(E.EngramError):            # output overlapping the input
        E.engram_ple_short_conv(x, w, dilation=3, group_size=64, out=x)
    with pytest.raises(E.EngramError):            # bf16 input, f16 output
        E.engram_ple_short_conv(x, w, dilation=3, group_size=64, out_dtype=torch.float16)


# ------------------------------------------------------------------- norm

@pytest.mark.parametrize("dt,out_dt,G", [("bf16", "bf16", 2560), ("bf16", "f32", 128),
                                         ("f16", "f16", 64), ("f32", "f32", 2048),
                                         ("f32", "f32", 8), ("bf16", "bf16", 4096),
                                         ("f32", "f32", 4096)])
def test_grouped_rms_norm(E, dt, out_dt, G):
    rows, C = 301, 4 * G if G <= 2048 else 2 * G
    x, nw, _, _ = small_inputs(dt, "bf16", rows, C, 1, 100 + G)
    out = E.engram_grouped_rms_norm(dev(x, dt), G, weight=dev(nw, "bf16"),
                                    out_dtype=TORCH_DT[out_dt])
    torch.cuda.synchronize()
    want = oracle.grouped_rms_norm(x, ORACLE_DT[dt], G, nw, oracle.BF16, 1e-6)
    assert_close(host(out), want, out_dt)


def test_grouped_rms_norm_in_place(E):
    rows, C, G = 1000, 5120, 2560
    x, nw, _, _ = small_inputs("bf16", "f32", rows, C, 1, 110)
    xt = dev(x, "bf16")
    E.engram_grouped_rms_norm(xt, G, weight=dev(nw, "f32"), out=xt)
    torch.cuda.synchronize()
    want = oracle.grouped_rms_norm(x, oracle.BF16, G, nw, oracle.F32, 1e-6)
    assert_close(host(xt), want, "bf16")


# ------------------------------------------------------- the page's shape

def test_page_shape_in_full(E):
    s = PLE_SHAPES["ple_full"]
    T, C = 2048, s.channels
    x, nw, w, b = small_inputs("bf16", "bf16", T, C, s.kernel, 120)
    cu = [0, 1024, 1500, 2048]
    got = run_conv(E, x, w, nw, b, cu, dt="bf16", wdt="bf16", out_dt="bf16", group=s.group,
                   dilation=s.dilation)
    want = oracle_conv(x, w, nw, b, cu, dt="bf16", wdt="bf16", group=s.group,
                       dilation=s.dilation)
    assert_close(got, want, "bf16")


def test_page_shape_benchmark_size_sampled(E):
    """The benchmark's launch: 16 x 4,096 tokens, C = 10,240 bf16. Sampled
    tokens (row starts and their first halo, block-range edges, the last
    token, random ones) are checked against the oracle run on the token and
    the 9 before it (clipped at its row start), which is all its output reads."""
    s = PLE_SHAPES["ple_full"]
    T, C, halo = s.tokens, s.channels, (s.kernel - 1) * s.dilation
    x, nw, w, b = ple_inputs(T, C, s.kernel, s.seed, "bf16")
    cu = row_bounds(s.batch, s.seq_len)
    out = E.engram_ple_short_conv(dev(x, "bf16"), dev(w, "bf16"), dilation=s.dilation,
                                  group_size=s.group, cu_seqlens=torch.from_numpy(cu).cuda(),
                                  norm_weight=dev(nw, "bf16"), conv_bias=dev(b, "bf16"))
    torch.cuda.synchronize()
    assert E.engram_get_device_error() == 0
    bpg = max(1, torch.cuda.get_device_properties(0).multi_processor_count // s.branches)
    rng = np.random.default_rng(7)
    sample = {0, 1, 2, 3, 8, 9, 10, T - 1, 4096, 4097, 4105, 4106, 12 * 4096 + 5}
    sample |= {T * j // bpg + d for j in range(bpg) for d in (-1, 0, 1) if 0 <= T * j // bpg + d < T}
    sample |= set(int(v) for v in rng.integers(0, T, 40))
    for t in sorted(sample):
        row0 = (t // s.seq_len) * s.seq_len
        w0 = max(row0, t - halo)
        want = oracle_conv(x[w0:t + 1], w, nw, b, None, dt="bf16", wdt="bf16", group=s.group,
                           dilation=s.dilation)[-1]
        got = out[t].float().cpu().numpy().astype(np.float64)
        assert_close(got, want, "bf16", f"token {t}")


@pytest.mark.parametrize("T,d", [(1, 3), (5, 9), (8, 4)])
def test_fewer_tokens_than_residues(E, T, d):
    # some residues of the dilation hold no token at all
    C, G = 128, 64
    x, nw, w, b = small_inputs("bf16", "f32", T, C, 4, 400 + T + d)
    got = run_conv(E, x, w, nw, b, None, dt="bf16", wdt="f32", out_dt="f32", group=G, dilation=d)
    want = oracle_conv(x, w, nw, b, None, dt="bf16", wdt="f32", group=G, dilation=d)
    assert_close(got, want, "f32", f"T={T} d={d}")
