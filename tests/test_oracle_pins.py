"""Pins for the fp64 oracle, each against something other than the oracle itself.

Anchors (none of the pages prints a numeric example, so these are the method's
stated properties, closed forms and an independent brute force):
  * softmax rows sum to one; weights times values ("FlashAttention by hand",
    conventional three-step computation);
  * deferred single division equals the per-step normalised form, and the tiled
    online update with rescaling equals the materialised softmax ("FlashAttention
    by hand", paragraphs on the running statistics, rescaling and the final
    division, and the closing remark on the two normalisation orders);
  * combining fragment statistics in any order or grouping gives the same exact
    result (ATTENTION2D, sections 2 and 3);
  * causal masking is part of the output stage (HOF SWIFT Attention, section 3,
    Transform).
Each case is chosen so that a plausible mistake fails it: a dropped max
subtraction, a wrong LSE base, an off-by-one causal test, a wrong offset sign, a
transposed operand, an interleaved head mapping, a missing final division.
"""

from __future__ import annotations

import itertools
import json
import math
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle
from workloads import randn_bf16

GOLDEN = Path(__file__).parent / "golden"


def bf16(x) -> torch.Tensor:
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def as4d(x):
    """[N, d] -> [1, 1, N, d]"""
    return x.reshape(1, 1, *x.shape)


# --------------------------------------------------------------------------------------
# independent brute force (long double, no max subtraction, direct sums)
# --------------------------------------------------------------------------------------
def brute_force(q, k, v, causal, scale, q_off=0, kv_off=0):
    ld = np.longdouble
    qd = q.to(torch.float64).numpy().astype(ld)
    kd = k.to(torch.float64).numpy().astype(ld)
    vd = v.to(torch.float64).numpy().astype(ld)
    B, Hq, Nq, d = qd.shape
    Hkv, Nkv = kd.shape[1], kd.shape[2]
    sc = ld(float(np.float32(scale)))
    O = np.zeros((B, Hq, Nq, d), dtype=ld)
    L = np.zeros((B, Hq, Nq), dtype=ld)
    for b in range(B):
        for h in range(Hq):
            g = (h * Hkv) // Hq
            for i in range(Nq):
                num = np.zeros(d, dtype=ld)
                den = ld(0)
                for j in range(Nkv):
                    if causal and kv_off + j > q_off + i:
                        continue
                    s = sc * np.sum(qd[b, h, i] * kd[b, g, j])
                    e = np.exp(s)
                    num += e * vd[b, g, j]
                    den += e
                if den == 0:
                    O[b, h, i] = 0
                    L[b, h, i] = -np.inf
                else:
                    O[b, h, i] = num / den
                    L[b, h, i] = np.log(den)
    return O.astype(np.float64), L.astype(np.float64)


def close(a, b, tol):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape
    ninf_a, ninf_b = np.isneginf(a), np.isneginf(b)
    assert np.array_equal(ninf_a, ninf_b), "-inf pattern differs"
    fin = ~ninf_a
    err = np.abs(a[fin] - b[fin]).max(initial=0.0)
    assert err <= tol, f"max abs diff {err} > {tol}"


# --------------------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal,q_off,kv_off", [(False, 0, 0), (True, 0, 0), (True, 5, 2),
                                                 (True, 3, 9)])
def test_softmax_rows_sum_to_one_and_output_is_weights_times_values(causal, q_off, kv_off):
    q = randn_bf16((2, 4, 9, 16), seed=11, tensor_id=0)
    k = randn_bf16((2, 2, 13, 16), seed=11, tensor_id=1)
    v = randn_bf16((2, 2, 13, 16), seed=11, tensor_id=2)
    o, lse, p = oracle.attention_rows(q, k, v, causal=causal, scale=0.3, q_off=q_off,
                                      kv_off=kv_off, want_p=True)
    assert (p >= 0).all()
    for b, h, i in itertools.product(range(2), range(4), range(9)):
        nvis = 13 if not causal else max(0, min(13, q_off + i - kv_off + 1))
        row = p[b, h, i]
        assert (row[nvis:] == 0).all()
        if nvis:
            assert abs(row.sum() - 1.0) <= 1e-12
            g = h // 2
            want = row @ v[b, g].to(torch.float64).numpy()
            assert np.abs(o[b, h, i] - want).max() <= 1e-12
        else:
            assert (o[b, h, i] == 0).all() and np.isneginf(lse[b, h, i])


def test_constant_values_give_that_value():
    q = randn_bf16((1, 2, 17, 32), seed=3, tensor_id=0)
    k = randn_bf16((1, 2, 23, 32), seed=3, tensor_id=1)
    c = randn_bf16((1, 2, 1, 32), seed=3, tensor_id=2)
    v = c.expand(1, 2, 23, 32).contiguous()
    for causal, q_off in [(False, 0), (True, 6)]:
        o, _ = oracle.attention(q, k, v, causal=causal, scale=0.7, q_off=q_off)
        want = np.broadcast_to(c.to(torch.float64).numpy(), o.shape)
        close(o, want, 1e-12)


def test_one_hot_dominant_logit_selects_one_value_row():
    N, d, t = 12, 8, 7
    qv = np.zeros((1, d)); qv[0, 0] = 8.0
    kv = np.zeros((N, d)); kv[t, 0] = 8.0            # logit 64 for key t, 0 elsewhere
    vv = np.arange(N * d, dtype=np.float32).reshape(N, d) / 16.0
    o, lse = oracle.attention(as4d(bf16(qv)), as4d(bf16(kv)), as4d(bf16(vv)), causal=False,
                              scale=1.0)
    assert np.abs(o[0, 0, 0] - vv[t]).max() <= 1e-20 + N * math.exp(-64) * np.abs(vv).max()
    assert abs(lse[0, 0, 0] - (64.0 + math.log1p((N - 1) * math.exp(-64)))) <= 1e-12


@pytest.mark.parametrize("causal,q_off,kv_off", [(False, 0, 0), (True, 0, 0), (True, 10, 4),
                                                 (True, 0, 7)])
def test_zero_scale_gives_mean_of_visible_values(causal, q_off, kv_off):
    Nq, Nkv = 11, 19
    q = randn_bf16((1, 3, Nq, 16), seed=5, tensor_id=0)
    k = randn_bf16((1, 3, Nkv, 16), seed=5, tensor_id=1)
    v = randn_bf16((1, 3, Nkv, 16), seed=5, tensor_id=2)
    o, lse = oracle.attention(q, k, v, causal=causal, scale=0.0, q_off=q_off, kv_off=kv_off)
    vd = v.to(torch.float64).numpy()
    for h in range(3):
        for i in range(Nq):
            n = Nkv if not causal else max(0, min(Nkv, q_off + i - kv_off + 1))
            if n == 0:
                assert np.isneginf(lse[0, h, i]) and (o[0, h, i] == 0).all()
            else:
                assert abs(lse[0, h, i] - math.log(n)) <= 1e-12
                assert np.abs(o[0, h, i] - vd[0, h, :n].mean(axis=0)).max() <= 1e-12


def test_identical_keys_give_mean_and_shifted_log_count():
    Nq, Nkv, d = 5, 9, 16
    q = randn_bf16((1, 1, Nq, d), seed=8, tensor_id=0)
    k1 = randn_bf16((1, 1, 1, d), seed=8, tensor_id=1)
    k = k1.expand(1, 1, Nkv, d).contiguous()
    v = randn_bf16((1, 1, Nkv, d), seed=8, tensor_id=2)
    o, lse = oracle.attention(q, k, v, causal=True, scale=0.25)
    qd, kd, vd = (t.to(torch.float64).numpy() for t in (q, k1, v))
    for i in range(Nq):
        s = 0.25 * float(qd[0, 0, i] @ kd[0, 0, 0])
        assert abs(lse[0, 0, i] - (s + math.log(i + 1))) <= 1e-12
        assert np.abs(o[0, 0, i] - vd[0, 0, : i + 1].mean(axis=0)).max() <= 1e-12


def test_single_key_and_causal_first_row():
    q = randn_bf16((1, 2, 6, 32), seed=9, tensor_id=0)
    k = randn_bf16((1, 2, 6, 32), seed=9, tensor_id=1)
    v = randn_bf16((1, 2, 6, 32), seed=9, tensor_id=2)
    qd, kd, vd = (t.to(torch.float64).numpy() for t in (q, k, v))
    o, lse = oracle.attention(q, k[:, :, :1].contiguous(), v[:, :, :1].contiguous(),
                              causal=False, scale=0.5)
    close(o, np.broadcast_to(vd[:, :, :1], o.shape), 0)
    close(lse, 0.5 * np.einsum("bhnd,bhd->bhn", qd, kd[:, :, 0]), 1e-12)
    o2, lse2 = oracle.attention(q, k, v, causal=True, scale=0.5)
    close(o2[:, :, 0], vd[:, :, 0], 0)
    close(lse2[:, :, 0], 0.5 * np.einsum("bhd,bhd->bh", qd[:, :, 0], kd[:, :, 0]), 1e-12)


def test_grouped_heads_read_contiguous_kv_groups():
    Hq, Hkv, N, d = 6, 2, 7, 8
    q = randn_bf16((1, Hq, N, d), seed=2, tensor_id=0)
    k = randn_bf16((1, Hkv, N, d), seed=2, tensor_id=1)
    v = torch.zeros((1, Hkv, N, d), dtype=torch.bfloat16)
    v[0, 1] = 1.0                                   # kv head index as the value
    o, _ = oracle.attention(q, k, v, causal=False, scale=0.4)
    for h in range(Hq):
        assert np.abs(o[0, h] - (h // 3)).max() <= 1e-12


def test_fully_masked_rows_are_zero_and_minus_inf():
    q = randn_bf16((1, 1, 8, 16), seed=4, tensor_id=0)
    k = randn_bf16((1, 1, 8, 16), seed=4, tensor_id=1)
    v = randn_bf16((1, 1, 8, 16), seed=4, tensor_id=2)
    o, lse = oracle.attention(q, k, v, causal=True, scale=0.25, q_off=0, kv_off=5)
    assert (o[0, 0, :5] == 0).all() and np.isneginf(lse[0, 0, :5]).all()
    assert np.isfinite(lse[0, 0, 5:]).all()


def test_large_logits_do_not_overflow():
    # logits 800 and 796: exp without max subtraction overflows a double
    q = bf16([[16.0, 0.0]])
    k = bf16([[50.0, 0.0], [49.75, 0.0], [0.0, 0.0]])    # 49.75 is exact in bf16
    assert float(k[1, 0]) == 49.75
    v = bf16([[1.0, 2.0], [3.0, -4.0], [5.0, 5.0]])
    o, lse = oracle.attention(as4d(q), as4d(k), as4d(v), causal=False, scale=1.0)
    s = [800.0, 796.0, 0.0]
    z = sum(math.exp(x - 800.0) for x in s)
    want = sum(math.exp(x - 800.0) * np.array(vv, dtype=float) for x, vv in
               zip(s, [[1, 2], [3, -4], [5, 5]])) / z
    assert np.abs(o[0, 0, 0] - want).max() <= 1e-12
    assert abs(lse[0, 0, 0] - (800.0 + math.log(z))) <= 1e-12


def test_scale_is_the_float_the_gpu_receives():
    q = randn_bf16((1, 1, 4, 16), seed=6, tensor_id=0)
    k = randn_bf16((1, 1, 4, 16), seed=6, tensor_id=1)
    v = randn_bf16((1, 1, 4, 16), seed=6, tensor_id=2)
    scale = 1.0 / math.sqrt(3.0)
    _, lse = oracle.attention(q, k, v, causal=False, scale=scale)
    _, lse_bf = brute_force(q, k, v, False, scale)
    close(lse, lse_bf, 1e-13)


# --------------------------------------------------------------------------------------
# hand-worked fixtures
# --------------------------------------------------------------------------------------
def _eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"exp": math.exp, "log": math.log}))


@pytest.mark.parametrize("case", json.loads((GOLDEN / "hand_worked.json").read_text())["cases"],
                         ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    q, k, v = (as4d(bf16(case[x])) for x in ("q", "k", "v"))
    assert torch.equal(q.float().reshape(-1), torch.tensor(case["q"]).reshape(-1))
    o, lse = oracle.attention(q, k, v, causal=case["causal"], scale=case["scale"])
    want_o = np.array([[_eval(e) for e in row] for row in case["expect_o"]])
    want_l = np.array([_eval(e) for e in case["expect_lse"]])
    assert np.abs(o[0, 0] - want_o).max() <= 1e-12
    assert np.abs(lse[0, 0] - want_l).max() <= 1e-12
    for tile in (1, 2, 3):
        o2, l2 = oracle.online_softmax_replay(q, k, v, causal=case["causal"],
                                              scale=case["scale"], tile=tile)
        assert np.abs(o2[0, 0] - want_o).max() <= 1e-12
        assert np.abs(l2[0, 0] - want_l).max() <= 1e-12


# --------------------------------------------------------------------------------------
# brute force on tiny inputs
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("Nq,Nkv,Hq,Hkv,causal,q_off,kv_off", [
    (1, 1, 1, 1, False, 0, 0), (5, 5, 2, 2, True, 0, 0), (7, 12, 4, 2, False, 0, 0),
    (12, 7, 4, 1, True, 3, 0), (16, 16, 2, 1, True, 0, 0), (9, 16, 3, 3, True, 20, 8),
    (16, 10, 2, 2, True, 0, 4)])
def test_brute_force_tiny(Nq, Nkv, Hq, Hkv, causal, q_off, kv_off):
    d = 8
    q = randn_bf16((2, Hq, Nq, d), seed=Nq * 31 + Nkv, tensor_id=0)
    k = randn_bf16((2, Hkv, Nkv, d), seed=Nq * 31 + Nkv, tensor_id=1)
    v = randn_bf16((2, Hkv, Nkv, d), seed=Nq * 31 + Nkv, tensor_id=2)
    o, lse = oracle.attention(q, k, v, causal=causal, scale=1 / math.sqrt(d), q_off=q_off,
                              kv_off=kv_off)
    ob, lb = brute_force(q, k, v, causal, 1 / math.sqrt(d), q_off, kv_off)
    close(o, ob, 1e-12)
    close(lse, lb, 1e-12)


# --------------------------------------------------------------------------------------
# online replay == materialised (deferred and per-step normalisation)
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("tile", [1, 3, 8, 64])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("normalise_each_step", [False, True])
def test_online_replay_equals_materialised(tile, causal, normalise_each_step):
    q = randn_bf16((1, 2, 33, 16), seed=tile, tensor_id=0)
    k = randn_bf16((1, 2, 40, 16), seed=tile, tensor_id=1)
    v = randn_bf16((1, 2, 40, 16), seed=tile, tensor_id=2)
    # rescale stress: large logits whose row maxima arrive late
    q = q * 8
    k[:, :, 31] *= 16
    k[:, :, 37] *= 16
    o, lse = oracle.attention(q, k, v, causal=causal, scale=0.25, q_off=7)
    o2, l2 = oracle.online_softmax_replay(q, k, v, causal=causal, scale=0.25, tile=tile,
                                          q_off=7, normalise_each_step=normalise_each_step)
    close(o2, o, 1e-12)
    close(l2, lse, 1e-12 * max(1.0, np.abs(lse[np.isfinite(lse)]).max()))


# --------------------------------------------------------------------------------------
# merge: chunked == unchunked, order and grouping independence, special cases
# --------------------------------------------------------------------------------------
def _chunkings(n):
    for mask in range(1 << (n - 1)):
        cuts = [0] + [i + 1 for i in range(n - 1) if mask >> i & 1] + [n]
        yield list(zip(cuts[:-1], cuts[1:]))


def _partials(q, k, v, causal, scale, chunks, q_off=0):
    parts = []
    for a, b in chunks:
        parts.append(oracle.attention(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(),
                                      causal=causal, scale=scale, q_off=q_off, kv_off=a))
    return parts


@pytest.mark.parametrize("causal,q_off", [(False, 0), (True, 0), (True, 3)])
def test_chunked_then_merged_equals_unchunked_exhaustive(causal, q_off):
    Nkv = 8
    q = randn_bf16((1, 2, 6, 8), seed=21, tensor_id=0)
    k = randn_bf16((1, 2, Nkv, 8), seed=21, tensor_id=1)
    v = randn_bf16((1, 2, Nkv, 8), seed=21, tensor_id=2)
    o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=0.4, q_off=q_off)
    for chunks in _chunkings(Nkv):
        parts = _partials(q, k, v, causal, 0.4, chunks, q_off)
        o, lse = oracle.merge([p[0] for p in parts], [p[1] for p in parts])
        close(o, o_ref, 1e-12)
        close(lse, l_ref, 1e-12)


def test_chunked_then_merged_equals_unchunked_random_16():
    rng = np.random.default_rng(0)
    q = randn_bf16((1, 2, 16, 8), seed=22, tensor_id=0) * 8
    k = randn_bf16((1, 2, 16, 8), seed=22, tensor_id=1)
    v = randn_bf16((1, 2, 16, 8), seed=22, tensor_id=2)
    for causal in (False, True):
        o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=0.35)
        for _ in range(40):
            mask = int(rng.integers(0, 1 << 15))
            cuts = [0] + [i + 1 for i in range(15) if mask >> i & 1] + [16]
            parts = _partials(q, k, v, causal, 0.35, list(zip(cuts[:-1], cuts[1:])))
            o, lse = oracle.merge([p[0] for p in parts], [p[1] for p in parts])
            close(o, o_ref, 1e-12)
            close(lse, l_ref, 1e-12 * np.abs(l_ref[np.isfinite(l_ref)]).max())


def test_merge_is_order_and_grouping_independent():
    q = randn_bf16((1, 2, 9, 8), seed=23, tensor_id=0) * 4
    k = randn_bf16((1, 2, 15, 8), seed=23, tensor_id=1)
    v = randn_bf16((1, 2, 15, 8), seed=23, tensor_id=2)
    chunks = [(0, 2), (2, 5), (5, 9), (9, 10), (10, 15)]
    parts = _partials(q, k, v, True, 0.5, chunks, q_off=6)
    o_ref, l_ref = oracle.merge([p[0] for p in parts], [p[1] for p in parts])
    for perm in itertools.permutations(range(5)):
        o, lse = oracle.merge([parts[i][0] for i in perm], [parts[i][1] for i in perm])
        close(o, o_ref, 1e-12)
        close(lse, l_ref, 1e-12)
    A, B, C = parts[0], oracle.merge([parts[1][0], parts[2][0]], [parts[1][1], parts[2][1]]), \
        oracle.merge([parts[3][0], parts[4][0]], [parts[3][1], parts[4][1]])
    left = oracle.merge([oracle.merge([A[0], B[0]], [A[1], B[1]])[0], C[0]],
                        [oracle.merge([A[0], B[0]], [A[1], B[1]])[1], C[1]])
    right_bc = oracle.merge([B[0], C[0]], [B[1], C[1]])
    right = oracle.merge([A[0], right_bc[0]], [A[1], right_bc[1]])
    close(left[0], right[0], 1e-12)
    close(left[1], right[1], 1e-12)
    close(left[0], o_ref, 1e-12)


def test_merge_special_cases():
    rng = np.random.default_rng(1)
    o1 = rng.standard_normal((3, 4))
    l1 = rng.standard_normal(3)
    o, lse = oracle.merge([o1], [l1])
    close(o, o1, 0)
    close(lse, l1, 0)
    empty_o, empty_l = np.zeros((3, 4)), np.full(3, -np.inf)
    o, lse = oracle.merge([empty_o, o1, empty_o], [empty_l, l1, empty_l])
    close(o, o1, 1e-15)
    close(lse, l1, 1e-15)
    o, lse = oracle.merge([empty_o, empty_o], [empty_l, empty_l])
    assert (o == 0).all() and np.isneginf(lse).all()
    # two equal-weight parts: the average, LSE + ln 2
    o, lse = oracle.merge([o1, -o1], [l1, l1])
    close(o, np.zeros_like(o1), 1e-15)
    close(lse, l1 + math.log(2.0), 1e-15)
