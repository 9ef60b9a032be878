"""Seeded random shapes for the PLE tail kernels against the oracle (B200).

Forty small configurations each for engram_ple_short_conv and
engram_ple_short_conv_backward: token counts 0..400 (often fewer than the
dilation's residues or a batch of rows), branch widths and counts, kernel
widths, dilations 1..16, random sequence layouts with empty and one-token
sequences, every flag combination and the three element types. The bars are
those of test_gpu_ple.py and test_gpu_ple_backward.py.
"""

import numpy as np
import pytest
import torch

import oracle
from tests.test_gpu_ple import assert_close
from tests.test_gpu_ple_backward import (ORACLE_DT, TORCH_DT, assert_dx, assert_wgrad, decode,
                                         dev, grad_input)
from workloads import ple_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    import hashed_gram_embedding_raw_b200 as E
    torch.cuda.set_device(0)
    E.engram_get_device_error()
    return E


def config(seed, backward):
    rng = np.random.default_rng(20_000 + seed + (1000 if backward else 0))
    G = int(rng.choice([8, 16, 24, 64, 136, 256, 520, 1280, 2560]))
    C = G * int(rng.integers(1, 4 if G <= 1280 else 2))
    K = int(rng.integers(1, 5 if backward else 9))
    d = int(rng.integers(1, 17))
    # widths above 4 take the chunked kernel, whose history must fit shared memory
    while K > 4 and 4 * G * ((K - 1) * d + 4) + 1152 > 227 * 1024:
        if d > 1:
            d //= 2
        else:
            G, C = 64, 128
    T = int(rng.choice([0, 1, 2, 3, 7, 9, 31, 64, 129, 257, 400]))
    if rng.random() < 0.5 or T == 0:
        cu = None
    else:
        n = int(rng.integers(1, 7))
        cuts = np.sort(rng.integers(0, T + 1, size=n - 1))
        cu = [0] + [int(v) for v in cuts] + [T]
    flags = tuple(int(v) for v in rng.integers(0, 2, size=3))
    dt = str(rng.choice(["bf16", "f16", "f32"]))
    gdt = str(rng.choice(["bf16", "f16", "f32"]))
    wdt = str(rng.choice(["bf16", "f16", "f32"]))
    return T, C, G, K, d, cu, flags, dt, gdt, wdt


def tensors(T, C, K, seed, dt, wdt):
    x, _, _, _ = ple_inputs(T, C, K, seed, dt)
    _, nw, w, b = ple_inputs(T, C, K, seed, wdt)
    return x, nw, w, b


@pytest.mark.parametrize("seed", range(40))
def test_forward(E, seed):
    T, C, G, K, d, cu, flags, dt, _, wdt = config(seed, False)
    out_dt = dt if seed % 2 else "f32"
    x, nw, w, b = tensors(T, C, K, seed, dt, wdt)
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    out = E.engram_ple_short_conv(dev(x, dt), dev(w, wdt), dilation=d, group_size=G,
                                  cu_seqlens=cu_t, norm_weight=dev(nw, wdt),
                                  conv_bias=dev(b, wdt), norm=bool(flags[0]),
                                  silu=bool(flags[1]), residual=bool(flags[2]),
                                  out_dtype=TORCH_DT[out_dt])
    torch.cuda.synchronize()
    assert E.engram_get_device_error() == 0
    want = oracle.short_conv(x, ORACLE_DT[dt], cu, w, dilation=d, group=G, norm_w=nw, eps=1e-6,
                             bias=b, wdtype=ORACLE_DT[wdt], norm=flags[0], silu=flags[1],
                             residual=flags[2])
    assert_close(out.float().cpu().numpy().astype(np.float64), want, out_dt,
                 f"T={T} C={C} G={G} K={K} d={d} cu={cu} flags={flags} {dt}/{wdt}")


@pytest.mark.parametrize("seed", range(40))
def test_backward(E, seed):
    T, C, G, K, d, cu, flags, dt, gdt, wdt = config(seed, True)
    x, nw, w, b = tensors(T, C, K, seed, dt, wdt)
    dout = grad_input(T, C, seed, gdt)
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    dx, dnw, dw, db = E.engram_ple_short_conv_backward(
        dev(x, dt), dev(w, wdt), dev(dout, gdt), dilation=d, group_size=G, cu_seqlens=cu_t,
        norm_weight=dev(nw, wdt), conv_bias=dev(b, wdt), norm=bool(flags[0]),
        silu=bool(flags[1]), residual=bool(flags[2]))
    torch.cuda.synchronize()
    assert E.engram_get_device_error() == 0
    want = oracle.short_conv_backward(x, ORACLE_DT[dt], cu, w, decode(dout, gdt), dilation=d,
                                      group=G, norm_w=nw, eps=1e-6, bias=b,
                                      wdtype=ORACLE_DT[wdt], norm=flags[0], silu=flags[1],
                                      residual=flags[2])
    what = f"T={T} C={C} G={G} K={K} d={d} cu={cu} flags={flags} {dt}/{gdt}/{wdt}"
    host = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    assert_dx(host(dx), want[0], gdt, what)
    for name, g_, w_ in zip(("dnorm_w", "dconv_w", "dbias"), (dnw, dw, db), want[1:]):
        assert_wgrad(host(g_), w_, f"{name} {what}")
