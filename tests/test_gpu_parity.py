"""GPU parity of attn_fwd, attn_fwd_partial and attn_merge against the fp64 oracle,
element by element, at sizes the oracle finishes quickly (several 128-row tiles and
ragged tails), plus edge cases. All calls go through the C ABI."""

from __future__ import annotations

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import MERGE_LSE_ULPS, TOL_MERGE, compare, to_np
from workloads import get, randn_bf16, attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def osx():
    import online_softmax_exact_b200 as m

    return m


def inputs(B, Hq, Hkv, Nq, Nkv, d, seed, q_mul=1.0, k_rows_mul=None):
    q = randn_bf16((B, Hq, Nq, d), seed, 0)
    k = randn_bf16((B, Hkv, Nkv, d), seed, 1)
    v = randn_bf16((B, Hkv, Nkv, d), seed, 2)
    if q_mul != 1.0:
        q = q * q_mul
    if k_rows_mul is not None:
        rows, mul = k_rows_mul
        k[:, :, rows] = k[:, :, rows] * mul
    return q, k, v


def run_fwd(osx, q, k, v, causal, scale):
    o, lse = osx.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    assert osx.attn_device_status() == osx.ATTN_OK
    return to_np(o), to_np(lse)


# ---------------------------------------------------------------------- tiny config
def test_tiny_config_fwd_partials_merge(osx):
    w = get("tiny_chunks4")
    q, k, v = attention_inputs(w)
    o_ref, l_ref = oracle.attention(q, k, v, causal=w.causal, scale=w.scale)
    o, lse = run_fwd(osx, q, k, v, w.causal, w.scale)
    compare(o, lse, o_ref, l_ref)

    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    C = w.N // w.n_chunks
    parts = []
    for c in range(w.n_chunks):
        op, lp = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=w.N, kv_start=c * C,
                                      kv_len=C, causal=w.causal, scale=w.scale)
        orf, lrf = oracle.attention(q, k[:, :, c * C:(c + 1) * C].contiguous(),
                                    v[:, :, c * C:(c + 1) * C].contiguous(), causal=w.causal,
                                    scale=w.scale, kv_off=c * C)
        compare(to_np(op), to_np(lp), orf, lrf)
        parts.append((op, lp))
    om, lm = osx.attn_merge([p[0] for p in parts], [p[1] for p in parts])
    # merge of identical fp32 partials vs the fp64 merge of the same partials
    o64, l64 = oracle.merge([to_np(p[0]) for p in parts], [to_np(p[1]) for p in parts])
    compare(to_np(om), to_np(lm), o64, l64, tol_o=TOL_MERGE, tol_lse=TOL_MERGE, lse_ulps=MERGE_LSE_ULPS)
    # chunked + merged vs the oracle, and vs the GPU single pass
    compare(to_np(om), to_np(lm), o_ref, l_ref)
    compare(to_np(om), to_np(lm), o, lse)


# ---------------------------------------------------------------------- shape sweep
SHAPES = [
    # B, Hq, Hkv, N, d, causal
    (1, 1, 1, 1, 64, False), (1, 1, 1, 1, 128, True), (1, 2, 2, 7, 64, True),
    (1, 2, 1, 16, 128, False), (2, 2, 2, 65, 64, True), (1, 4, 2, 129, 128, True),
    (1, 2, 2, 257, 128, False), (2, 8, 1, 300, 64, True), (1, 4, 4, 600, 128, True),
    (1, 8, 2, 513, 128, False), (1, 2, 2, 1000, 64, False), (1, 16, 2, 384, 128, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", SHAPES,
                         ids=lambda x: str(x))
def test_fwd_shapes(osx, B, Hq, Hkv, N, d, causal):
    q, k, v = inputs(B, Hq, Hkv, N, N, d, seed=N * 7 + d + Hq)
    scale = 1 / math.sqrt(d)
    o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=scale)
    o, lse = run_fwd(osx, q, k, v, causal, scale)
    compare(o, lse, o_ref, l_ref)


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_rescale_stress(osx, d):
    """Q*8 and a few K rows *16: logits in the hundreds, maxima that arrive late."""
    N = 700
    rows = torch.tensor([5, 170, 333, 512, 690])
    q, k, v = inputs(1, 4, 4, N, N, d, seed=99, q_mul=8.0, k_rows_mul=(rows, 16.0))
    for causal in (False, True):
        o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=1 / math.sqrt(d))
        o, lse = run_fwd(osx, q, k, v, causal, 1 / math.sqrt(d))
        compare(o, lse, o_ref, l_ref)


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_running_max_jumps(osx, d):
    """Rows whose maximum jumps by tens of octaves (P rescaled in place by a power of
    two) and by hundreds (P recomputed) on later key tiles, with and without the mask."""
    N = 640
    q, k, v = inputs(1, 2, 2, N, N, d, seed=123)
    q = q.clone()
    k = k.clone()
    q[..., 0] = 8.0
    # with q[0] = 8, k[0] = J ln2 sqrt(d) / 8 lifts that key's logit by about J octaves
    # (the others stay within a few octaves of 0)
    for j, octaves in ((200, 30.0), (250, 60.0), (400, 200.0), (600, 800.0)):
        k[:, :, j, 0] = octaves * math.log(2.0) * math.sqrt(d) / 8.0
    for causal in (False, True):
        o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=1 / math.sqrt(d))
        o, lse = run_fwd(osx, q, k, v, causal, 1 / math.sqrt(d))
        compare(o, lse, o_ref, l_ref)


def test_fwd_zero_scale_is_mean_of_visible_values(osx):
    q, k, v = inputs(1, 2, 2, 300, 300, 128, seed=5)
    o, lse = run_fwd(osx, q, k, v, True, 0.0)
    vd = v.to(torch.float64).numpy()
    want = np.cumsum(vd, axis=2) / np.arange(1, 301)[None, None, :, None]
    assert np.abs(o - want).max() <= 2e-2
    assert np.abs(lse - np.log(np.arange(1, 301))[None, None]).max() <= 5e-3


# ---------------------------------------------------------------------- partials
PARTIALS = [
    # Lq, Lkv, q_start, q_len, kv_start, kv_len, q_off, kv_off, causal, d
    (512, 512, 128, 256, 0, 384, None, None, True, 128),    # kv chunk straddles the diagonal
    (512, 512, 0, 256, 256, 256, None, None, True, 128),    # kv after q: every row masked
    (512, 512, 256, 256, 0, 256, None, None, True, 64),     # kv before q: no mask needed
    (600, 700, 100, 300, 37, 450, None, None, False, 64),   # ragged, unaligned starts
    (600, 700, 100, 300, 37, 450, 1000, 1200, True, 128),   # explicit global offsets
    (300, 300, 0, 300, 0, 1, None, None, False, 128),       # one key
    (1024, 1024, 512, 512, 384, 256, None, None, True, 64),  # partly masked rows
]


@pytest.mark.parametrize("case", PARTIALS, ids=lambda x: str(x))
def test_fwd_partial(osx, case):
    Lq, Lkv, qs, ql, ks, kl, q_off, kv_off, causal, d = case
    q, k, v = inputs(1, 4, 2, Lq, Lkv, d, seed=Lq + Lkv + qs + ks)
    scale = 1 / math.sqrt(d)
    qo = qs if q_off is None else q_off
    ko = ks if kv_off is None else kv_off
    o, lse = osx.attn_fwd_partial(q.cuda(), k.cuda(), v.cuda(), q_start=qs, q_len=ql,
                                  kv_start=ks, kv_len=kl, causal=causal, scale=scale,
                                  q_off=qo, kv_off=ko)
    assert osx.attn_device_status() == osx.ATTN_OK
    o_ref, l_ref = oracle.attention(q[:, :, qs:qs + ql].contiguous(),
                                    k[:, :, ks:ks + kl].contiguous(),
                                    v[:, :, ks:ks + kl].contiguous(), causal=causal,
                                    scale=scale, q_off=qo, kv_off=ko)
    compare(to_np(o), to_np(lse), o_ref, l_ref)


# ---------------------------------------------------------------------- merge
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 9, 17, 64])
def test_merge_random_parts(osx, n, d):
    g = torch.Generator().manual_seed(n * 1000 + d)
    rows = 1000
    o_parts = [torch.randn((rows, d), generator=g) for _ in range(n)]
    l_parts = [torch.randn((rows,), generator=g) * 30 for _ in range(n)]
    # some rows empty in some parts, some rows empty in all parts
    for i in range(n):
        dead = torch.rand(rows, generator=g) < 0.2
        dead[:7] = True
        l_parts[i][dead] = -math.inf
        o_parts[i][dead] = 0.0
    og = [t.cuda() for t in o_parts]
    lg = [t.cuda() for t in l_parts]
    om, lm = osx.attn_merge(og, lg)
    o64, l64 = oracle.merge([t.double().numpy() for t in o_parts],
                            [t.double().numpy() for t in l_parts])
    compare(to_np(om), to_np(lm), o64, l64, tol_o=TOL_MERGE, tol_lse=TOL_MERGE, lse_ulps=MERGE_LSE_ULPS)
    assert (to_np(om)[:7] == 0).all() and np.isneginf(to_np(lm)[:7]).all()


def test_merge_order_and_grouping_on_gpu(osx):
    q, k, v = inputs(1, 4, 4, 512, 512, 128, seed=17)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    bounds = [(0, 100), (100, 256), (256, 300), (300, 512)]
    parts = [osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=512, kv_start=a, kv_len=b - a,
                                  causal=True, scale=128 ** -0.5) for a, b in bounds]
    ref = osx.attn_merge([p[0] for p in parts], [p[1] for p in parts])
    for perm in itertools.permutations(range(4)):
        om, lm = osx.attn_merge([parts[i][0] for i in perm], [parts[i][1] for i in perm])
        compare(to_np(om), to_np(lm), to_np(ref[0]), to_np(ref[1]), tol_o=TOL_MERGE,
                tol_lse=TOL_MERGE, lse_ulps=MERGE_LSE_ULPS)
    ab = osx.attn_merge([parts[0][0], parts[1][0]], [parts[0][1], parts[1][1]])
    cd = osx.attn_merge([parts[2][0], parts[3][0]], [parts[2][1], parts[3][1]])
    grouped = osx.attn_merge([ab[0], cd[0]], [ab[1], cd[1]])
    compare(to_np(grouped[0]), to_np(grouped[1]), to_np(ref[0]), to_np(ref[1]),
            tol_o=1e-5, tol_lse=1e-5, lse_ulps=MERGE_LSE_ULPS)
    o_ref, l_ref = oracle.attention(q, k, v, causal=True, scale=128 ** -0.5)
    compare(to_np(ref[0]), to_np(ref[1]), o_ref, l_ref)
    single = osx.attn_fwd(qg, kg, vg, causal=True, scale=128 ** -0.5)
    do, dl = compare(to_np(ref[0]), to_np(ref[1]), to_np(single[0]), to_np(single[1]))
    print(f"chunked+merged vs single pass on GPU: max|dO|={do:.2e} max|dLSE|={dl:.2e}")


# ---------------------------------------------------------------------- errors
def test_invalid_arguments_return_status(osx):
    q = torch.zeros((1, 2, 64, 64), dtype=torch.bfloat16, device="cuda")
    k3 = torch.zeros((1, 3, 64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(osx.AttnError) as e:
        osx.attn_fwd(q, k3, k3, causal=False)
    assert e.value.status == osx.ATTN_ERR_INVALID_ARG
    o = torch.empty((1, 2, 64, 64), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 2, 64), dtype=torch.float32, device="cuda")
    lib = osx.lib()
    # Hq % Hkv != 0
    assert lib.attn_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(),
                        1, 2, 3, 64, 64, 0, 0.125, None) == osx.ATTN_ERR_INVALID_ARG
    # unsupported head dim
    assert lib.attn_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(),
                        1, 2, 2, 64, 96, 0, 0.125, None) == osx.ATTN_ERR_UNSUPPORTED
    # output aliasing an input
    assert lib.attn_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), lse.data_ptr(),
                        1, 2, 2, 64, 64, 0, 0.125, None) == osx.ATTN_ERR_INVALID_ARG


def test_injected_failure_launches_nothing(osx):
    q = torch.randn((1, 2, 64, 64), device="cuda").to(torch.bfloat16)
    before = osx.attn_launch_count()
    osx.attn_debug_inject(osx.ATTN_ERR_INJECTED, 1)
    with pytest.raises(osx.AttnError) as e:
        osx.attn_fwd(q, q, q, causal=False)
    assert e.value.status == osx.ATTN_ERR_INJECTED
    assert osx.attn_launch_count() == before
    osx.attn_fwd(q, q, q, causal=False)          # next call runs again
    assert osx.attn_launch_count() == before + 1
    assert osx.attn_device_status() == osx.ATTN_OK
