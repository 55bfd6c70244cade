"""Pins for the fp64 oracle: values the pages print, closed forms, invariants, brute force on
tiny inputs and an independent library computation. None of these re-types the oracle's own
formula; each is chosen so that a plausible slip (dropped term, wrong sign, transposed operand,
wrong index or scale) fails at least one of them."""
import json
import math
import os

import numpy as np
import pytest
import torch

import attn_inputs
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return (g.standard_normal(shape) * scale).astype(np.float32)


# --------------------------------------------------------------------------------------------
# Score-matrix size ("Calculateur de mémoire d'attention", "La formule" / "Exemple chiffré";
# "Efficient Attention", printed output of efficient_attention.py)
# --------------------------------------------------------------------------------------------
def test_score_bytes_match_printed_values():
    gold = json.load(open(os.path.join(GOLDEN, "score_matrix_bytes.json")))
    for e in gold["exact"]:
        assert oracle.score_matrix_bytes(e["B"], e["H"], e["n"], e["e"]) == e["bytes"], e["cite"]
    for e in gold["approximate"]:
        got = oracle.score_matrix_bytes(e["B"], e["H"], e["n"], e["e"]) / e["unit"]
        assert round(got, e["digits"]) == pytest.approx(e["value"]), e["cite"]
    rb = gold["row_block"]
    block = rb["block_rows"] * rb["n"] * rb["e"]
    assert block == rb["block_bytes"]
    assert oracle.score_matrix_bytes(1, 1, rb["n"], rb["e"]) // block == rb["ratio"]


def test_score_bytes_quadratic_growth():
    # "4x panjang seq -> 16x memori skor" (Efficient Attention, printed output)
    assert oracle.score_matrix_bytes(1, 1, 4000, 4) == 16 * oracle.score_matrix_bytes(1, 1, 1000, 4)
    # doubling the context quadruples the matrix (Calculateur, "Exemple chiffré")
    assert oracle.score_matrix_bytes(1, 32, 8192, 2) == 4 * oracle.score_matrix_bytes(1, 32, 4096, 2)


# --------------------------------------------------------------------------------------------
# Forward: brute force and closed forms
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_single_key_returns_value_and_score(causal):
    q, k, v = _rand((1, 2, 1, 8), 1), _rand((1, 2, 1, 8), 2), _rand((1, 2, 1, 8), 3)
    o, lse = oracle.fwd(q, k, v, 0.37, causal)
    np.testing.assert_array_equal(o, v.astype(np.float64))
    want = 0.37 * np.sum(q.astype(np.float64) * k.astype(np.float64), axis=-1)
    np.testing.assert_allclose(lse, want, rtol=0, atol=1e-15)


def test_two_keys_brute_force():
    q, k, v = _rand((1, 1, 2, 4), 4), _rand((1, 1, 2, 4), 5), _rand((1, 1, 2, 4), 6)
    scale = 0.5
    o, lse = oracle.fwd(q, k, v, scale, False)
    oc, lsec = oracle.fwd(q, k, v, scale, True)
    Q, K, V = (x[0, 0].astype(np.float64) for x in (q, k, v))
    for i in range(2):
        s0 = scale * sum(Q[i][c] * K[0][c] for c in range(4))
        s1 = scale * sum(Q[i][c] * K[1][c] for c in range(4))
        w1 = 1.0 / (1.0 + math.exp(s0 - s1))          # softmax of two scores is a sigmoid
        want = [(1 - w1) * V[0][c] + w1 * V[1][c] for c in range(4)]
        np.testing.assert_allclose(o[0, 0, i], want, rtol=0, atol=1e-14)
        assert lse[0, 0, i] == pytest.approx(math.log(math.exp(s0) + math.exp(s1)), abs=1e-14)
    # causal: row 0 sees only key 0, row 1 sees both
    np.testing.assert_array_equal(oc[0, 0, 0], V[0])
    s00 = scale * float(np.dot(Q[0], K[0]))
    assert lsec[0, 0, 0] == pytest.approx(s00, abs=1e-15)
    np.testing.assert_allclose(oc[0, 0, 1], o[0, 0, 1], rtol=0, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_identity_values_expose_probabilities(causal):
    # With V = I (n = d), O is the probability matrix itself: rows sum to 1 ("Attention
    # Mechanism ...", §3 Step 3), entries are >= 0, and the causal mask zeroes j > i (§4.4).
    n = 24
    q, k = _rand((1, 1, n, n), 7), _rand((1, 1, n, n), 8)
    v = np.eye(n, dtype=np.float32).reshape(1, 1, n, n)
    P, lse = oracle.fwd(q, k, v, 0.3, causal)
    P = P[0, 0]
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-14)
    assert (P >= 0).all()
    if causal:
        assert np.all(np.triu(P, 1) == 0.0)
        assert np.all(np.diag(P) > 0)
    # the row with the largest score gets the largest weight, and P = exp(S - lse)
    S = 0.3 * q[0, 0].astype(np.float64) @ k[0, 0].astype(np.float64).T
    if causal:
        S = np.where(np.tril(np.ones((n, n), bool)), S, -np.inf)
    np.testing.assert_allclose(P, np.exp(S - lse[0, 0][:, None]), rtol=1e-13, atol=1e-300)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_return_that_row(causal):
    q, k = _rand((2, 2, 40, 16), 9), _rand((2, 2, 40, 16), 10)
    row = _rand((16,), 11)
    v = np.broadcast_to(row, (2, 2, 40, 16)).copy()
    o, _ = oracle.fwd(q, k, v, 0.25, causal)
    np.testing.assert_allclose(o, np.broadcast_to(row.astype(np.float64), o.shape), rtol=0,
                               atol=1e-14)


def test_zero_queries_give_mean_and_log_n():
    n, d = 37, 8
    q = np.zeros((1, 1, n, d), np.float32)
    k, v = _rand((1, 1, n, d), 12), _rand((1, 1, n, d), 13)
    V = v[0, 0].astype(np.float64)
    o, lse = oracle.fwd(q, k, v, 1.0, False)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(V.mean(0), (n, d)), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], math.log(n), rtol=0, atol=1e-14)
    oc, lsec = oracle.fwd(q, k, v, 1.0, True)
    prefix = np.cumsum(V, 0) / np.arange(1, n + 1)[:, None]
    np.testing.assert_allclose(oc[0, 0], prefix, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lsec[0, 0], np.log(np.arange(1, n + 1)), rtol=0, atol=1e-14)


def test_causal_edge_rows():
    q, k, v = (_rand((1, 3, 50, 16), s) for s in (14, 15, 16))
    oc, lsec = oracle.fwd(q, k, v, 0.25, True)
    o, lse = oracle.fwd(q, k, v, 0.25, False)
    np.testing.assert_array_equal(oc[:, :, 0], v[:, :, 0].astype(np.float64))
    np.testing.assert_allclose(oc[:, :, -1], o[:, :, -1], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lsec[:, :, -1], lse[:, :, -1], rtol=0, atol=1e-13)
    # row i of the causal result depends only on keys/values 0..i
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 30:] = 5.0
    v2[:, :, 30:] = -3.0
    oc2, _ = oracle.fwd(q, k2, v2, 0.25, True)
    np.testing.assert_array_equal(oc2[:, :, :30], oc[:, :, :30])


def test_key_shift_invariance():
    # Adding u to every key adds scale*q_i.u to every score of row i: O is unchanged and the
    # log-sum-exp moves by exactly that amount. A transposed Q/K or a per-column softmax fails.
    q, k, v = (_rand((1, 2, 33, 8), s) for s in (17, 18, 19))
    u = _rand((8,), 20)
    # dyadic values with few bits, so that k + u is exact in fp32
    k = np.round(k * 1024) / 1024
    u = (np.round(u * 1024) / 1024).astype(np.float32)
    k = k.astype(np.float32)
    o, lse = oracle.fwd(q, k, v, 0.4, False)
    o2, lse2 = oracle.fwd(q, k + u, v, 0.4, False)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    shift = 0.4 * (q.astype(np.float64) @ u.astype(np.float64))
    np.testing.assert_allclose(lse2 - lse, shift, rtol=0, atol=1e-12)


def test_large_inputs_stay_finite():
    q, k, v = (_rand((1, 1, 64, 32), s, 30.0) for s in (21, 22, 23))
    for causal in (False, True):
        o, lse = oracle.fwd(q, k, v, 1 / math.sqrt(32), causal)
        assert np.isfinite(o).all() and np.isfinite(lse).all()
        assert np.abs(o).max() <= np.abs(v).max() + 1e-9   # convex combination of value rows


# --------------------------------------------------------------------------------------------
# Row tiling and the online-softmax recurrence
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [128, 100, 1])
def test_rowtiled_equals_full_bitwise(causal, block):
    # "Efficient Attention": per-128-row blocks give torch.equal results (printed "True").
    q, k, v = (_rand((1, 2, 300, 32), s) for s in (24, 25, 26))
    o, lse = oracle.fwd(q, k, v, 0.17, causal)
    ot, lset = oracle.fwd_rowtiled(q, k, v, 0.17, causal, block)
    assert np.array_equal(o, ot) and np.array_equal(lse, lset)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [128, 64, 7])
def test_online_softmax_matches_definition(causal, block):
    q, k, v = (_rand((2, 2, 333, 32), s, 2.0) for s in (27, 28, 29))
    o, lse = oracle.fwd(q, k, v, 0.2, causal)
    oo, lseo = oracle.fwd_online(q, k, v, 0.2, causal, block)
    np.testing.assert_allclose(oo, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lseo, lse, rtol=0, atol=1e-12)


def test_printed_online_update_is_wrong_when_max_moves():
    # The O update as printed in §13 of "Attention Mechanism ..." lacks exp(m_old - m_new) on
    # the old term. With several KV blocks the running max moves and the printed form drifts;
    # with a single block it is exact (no rescaling happens).
    q, k, v = (_rand((1, 1, 256, 32), s, 2.0) for s in (30, 31, 32))
    o, _ = oracle.fwd(q, k, v, 0.2, False)
    lit, _ = oracle.fwd_online(q, k, v, 0.2, False, 32, literal_page_form=True)
    assert np.abs(lit - o).max() > 1e-2
    one, _ = oracle.fwd_online(q, k, v, 0.2, False, 256, literal_page_form=True)
    np.testing.assert_allclose(one, o, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------------------------
# Independent computation with torch fp64 CPU ops (a library routine, not the oracle's loops)
# --------------------------------------------------------------------------------------------
def _torch_ref(q, k, v, scale, causal):
    Q, K, V = (torch.from_numpy(x.astype(np.float64)) for x in (q, k, v))
    S = Q @ K.transpose(-1, -2) * scale
    if causal:
        n = S.shape[-1]
        S = S.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    return (torch.softmax(S, -1) @ V).numpy(), torch.logsumexp(S, -1).numpy()


@pytest.mark.parametrize("shape,causal", [((2, 3, 70, 16), False), ((1, 2, 129, 64), True),
                                          ((1, 1, 5, 128), True), ((2, 1, 200, 32), False)])
def test_matches_torch_fp64(shape, causal):
    q, k, v = (_rand(shape, s) for s in (33, 34, 35))
    scale = 1 / math.sqrt(shape[-1])
    o, lse = oracle.fwd(q, k, v, scale, causal)
    ro, rlse = _torch_ref(q, k, v, scale, causal)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, rlse, rtol=0, atol=1e-12)


def test_p1_manual_fp32_agrees_within_page_tolerance():
    # "Efficient Attention": the fp32 manual path (q@k^T/sqrt(d), softmax, @v) matches the fused
    # result within atol 1e-5 (printed: max diff 8.34e-07, allclose True). The fp64 oracle must
    # agree with that fp32 manual path at the same tolerance, on the same seed-9 draws.
    (q, k, v), _ = attn_inputs.p1_script_draws()
    manual = (q @ k.transpose(-2, -1) / math.sqrt(32)).softmax(dim=-1) @ v
    o, _ = oracle.fwd(q, k, v, 1 / math.sqrt(32), False)
    err = np.abs(o - manual.double().numpy()).max()
    assert err < 1e-5
    assert err > 0.0   # fp32 vs fp64 cannot agree exactly on 12k outputs


# --------------------------------------------------------------------------------------------
# Sampled-row entry points reproduce the full computation row for row
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_equal_full(causal):
    q, k, v, do = (_rand((2, 2, 150, 32), s) for s in (36, 37, 38, 39))
    o, lse = oracle.fwd(q, k, v, 0.18, causal)
    rows = [0, 5, 149, 150, 299, 451, 599]
    ro, rl = oracle.fwd_rows(q, k, v, 0.18, causal, rows)
    np.testing.assert_array_equal(ro, o.reshape(-1, 32)[rows])
    np.testing.assert_array_equal(rl, lse.reshape(-1)[rows])
    dq, dk, dv, D = oracle.bwd(q, k, v, do, 0.18, causal)
    rq, rD = oracle.bwd_query_rows(q, k, v, do, 0.18, causal, rows)
    np.testing.assert_allclose(rq, dq.reshape(-1, 32)[rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(rD, D.reshape(-1)[rows], rtol=0, atol=1e-14)
    keys = [0, 17, 77, 149]
    for bh in (0, 3):
        kk, vv = oracle.bwd_key_rows(q, k, v, do, 0.18, causal, bh, keys)
        np.testing.assert_allclose(kk, dk.reshape(4, 150, 32)[bh][keys], rtol=0, atol=1e-13)
        np.testing.assert_allclose(vv, dv.reshape(4, 150, 32)[bh][keys], rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_batched_key_rows_equal_full(causal):
    # The batched form (matrix products over 64-row batches, a ragged last batch of 44 rows)
    # reproduces the loop oracle's full backward at keys on both sides of batch edges.
    q, k, v, do = (_rand((2, 2, 300, 32), s) for s in (60, 61, 62, 63))
    dq, dk, dv, _ = oracle.bwd(q, k, v, do, 0.18, causal)
    keys = [0, 1, 63, 64, 150, 256, 299]
    for bh in (0, 3):
        kk, vv = oracle.bwd_key_rows_batched(q, k, v, do, 0.18, causal, bh, keys, block_rows=64)
        np.testing.assert_allclose(kk, dk.reshape(4, 300, 32)[bh][keys], rtol=0, atol=1e-12)
        np.testing.assert_allclose(vv, dv.reshape(4, 300, 32)[bh][keys], rtol=0, atol=1e-12)


def test_batched_key_rows_match_autograd_fp64():
    # Independent of the loop oracle: torch fp64 autograd of the causal definition.
    q, k, v, do = (_rand((1, 2, 70, 8), s) for s in (64, 65, 66, 67))
    scale = 0.4
    Q, K, V = (torch.from_numpy(x.astype(np.float64)).requires_grad_() for x in (q, k, v))
    S = (Q @ K.transpose(-1, -2) * scale).masked_fill(
        torch.ones(70, 70, dtype=torch.bool).triu(1), float("-inf"))
    (torch.softmax(S, -1) @ V).backward(torch.from_numpy(do.astype(np.float64)))
    keys = [0, 15, 16, 40, 69]
    kk, vv = oracle.bwd_key_rows_batched(q, k, v, do, scale, True, 1, keys, block_rows=16)
    np.testing.assert_allclose(kk, K.grad.numpy()[0, 1][keys], rtol=0, atol=1e-12)
    np.testing.assert_allclose(vv, V.grad.numpy()[0, 1][keys], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------------------------
# Backward: autograd fp64, finite differences, invariants
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_autograd_fp64(causal):
    q, k, v, do = (_rand((2, 3, 16, 8), s) for s in (40, 41, 42, 43))
    scale = 0.35
    dq, dk, dv, D = oracle.bwd(q, k, v, do, scale, causal)
    Q, K, V = (torch.from_numpy(x.astype(np.float64)).requires_grad_() for x in (q, k, v))
    S = Q @ K.transpose(-1, -2) * scale
    if causal:
        S = S.masked_fill(torch.ones(16, 16, dtype=torch.bool).triu(1), float("-inf"))
    O = torch.softmax(S, -1) @ V
    O.backward(torch.from_numpy(do.astype(np.float64)))
    np.testing.assert_allclose(dq, Q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, K.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, V.grad.numpy(), rtol=0, atol=1e-12)
    # D_i = sum_j P_ij dP_ij equals rowsum(dO ∘ O)
    np.testing.assert_allclose(D, (do.astype(np.float64) * O.detach().numpy()).sum(-1), rtol=0,
                               atol=1e-13)


def test_backward_finite_differences():
    # Central differences of L = sum(O ∘ G) with respect to a few entries of Q, K and V.
    q, k, v, g = (_rand((1, 1, 6, 4), s) for s in (44, 45, 46, 47))
    scale, h = 0.6, 1e-3
    for causal in (False, True):
        dq, dk, dv, _ = oracle.bwd(q, k, v, g, scale, causal)

        def loss(qq, kk, vv):
            o, _ = oracle.fwd(qq, kk, vv, scale, causal)
            return float((o * g.astype(np.float64)).sum())

        for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            for idx in [(0, 0, 0, 0), (0, 0, 3, 2), (0, 0, 5, 3)]:
                plus, minus = arr.copy(), arr.copy()
                # finite-difference steps applied to fp32 inputs: use the realised step
                plus[idx] += h
                minus[idx] -= h
                step = float(plus[idx]) - float(minus[idx])
                args_p = {"q": q, "k": k, "v": v}
                args_m = dict(args_p)
                args_p[name], args_m[name] = plus, minus
                fd = (loss(args_p["q"], args_p["k"], args_p["v"]) -
                      loss(args_m["q"], args_m["k"], args_m["v"])) / step
                assert fd == pytest.approx(grad[idx], abs=2e-6), (name, idx, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    q, k, v, do = (_rand((1, 2, 90, 16), s) for s in (48, 49, 50, 51))
    dq, dk, dv, _ = oracle.bwd(q, k, v, do, 0.25, causal)
    # each dS row sums to 0 -> sum over keys of dK vanishes
    np.testing.assert_allclose(dk.sum(2), 0.0, rtol=0, atol=1e-12)
    # each P row sums to 1 -> sum over keys of dV equals sum over queries of dO
    np.testing.assert_allclose(dv.sum(2), do.astype(np.float64).sum(2), rtol=0, atol=1e-12)
    if causal:
        # the last key is seen only by the last query: dV_{n-1} = P_{n-1,n-1} dO_{n-1}
        _, lse = oracle.fwd(q, k, v, 0.25, True)
        s = 0.25 * np.sum(q[:, :, -1].astype(np.float64) * k[:, :, -1], -1)
        p = np.exp(s - lse[:, :, -1])
        np.testing.assert_allclose(dv[:, :, -1], p[..., None] * do[:, :, -1], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------------------------
# Workload draws (the seed-9 stream of efficient_attention.py)
# --------------------------------------------------------------------------------------------
def test_p1_draws_shapes_and_stream():
    (q, k, v), (q2, k2, v2) = attn_inputs.p1_script_draws()
    assert tuple(q.shape) == (2, 3, 128, 32) and tuple(q2.shape) == (4096, 64)
    # the score tensor of the first block is (2,3,128,128) fp32 = 393,216 bytes (printed)
    assert q.shape[0] * q.shape[1] * q.shape[2] * k.shape[2] * 4 == 393216
    (qa, _, _), (q2a, _, _) = attn_inputs.p1_script_draws()
    assert torch.equal(q, qa) and torch.equal(q2, q2a)
    assert not torch.equal(q, k)


def test_bf16_draws_are_rounded_and_reproducible():
    a = attn_inputs.bf16_draws((1, 2, 8, 16), factor=0.5)
    b = attn_inputs.bf16_draws((1, 2, 8, 16), factor=0.5)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert all(x.dtype == torch.bfloat16 for x in a)
    assert float(a[0].float().abs().max()) < 4.0


# --------------------------------------------------------------------------------------------
# Grouped-query attention ("Attention Mechanism ...", §12 "GQA vs MQA")
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_with_all_kv_heads_is_mha(causal):
    q, k, v, do = (_rand((2, 4, 40, 16), s) for s in (60, 61, 62, 63))
    o, lse = oracle.fwd(q, k, v, 0.25, causal)
    og, lseg = oracle.fwd_gqa(q, k, v, 0.25, causal)
    assert np.array_equal(o, og) and np.array_equal(lse, lseg)
    ref = oracle.bwd(q, k, v, do, 0.25, causal)
    got = oracle.bwd_gqa(q, k, v, do, 0.25, causal)
    for a, b in zip(ref, got):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("Hkv,causal", [(2, False), (2, True), (1, True)])
def test_gqa_matches_torch_repeat_interleave_autograd(Hkv, causal):
    # The page's recipe, run by torch in fp64 with autograd: repeat_interleave(g, dim=1), then
    # standard attention; gradients flow back through the repeat into the shared K/V heads.
    H, n, d, scale = 4, 12, 8, 0.3
    q, do = _rand((1, H, n, d), 64), _rand((1, H, n, d), 65)
    k, v = _rand((1, Hkv, n, d), 66), _rand((1, Hkv, n, d), 67)
    Q, K, V = (torch.from_numpy(x.astype(np.float64)).requires_grad_() for x in (q, k, v))
    g = H // Hkv
    S = Q @ K.repeat_interleave(g, dim=1).transpose(-1, -2) * scale
    if causal:
        S = S.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    O = torch.softmax(S, -1) @ V.repeat_interleave(g, dim=1)
    O.backward(torch.from_numpy(do.astype(np.float64)))
    o, _ = oracle.fwd_gqa(q, k, v, scale, causal)
    dq, dk, dv, _ = oracle.bwd_gqa(q, k, v, do, scale, causal)
    np.testing.assert_allclose(o, O.detach().numpy(), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dq, Q.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, K.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, V.grad.numpy(), rtol=0, atol=1e-12)


def test_mqa_heads_with_equal_queries_agree():
    # MQA (one K/V head): query heads with identical queries give identical outputs, and the
    # shared dV is the sum over heads of P^T dO (here: H times one head's dV for equal dO)
    qh, doh = _rand((1, 1, 30, 8), 68), _rand((1, 1, 30, 8), 69)
    q, do = np.repeat(qh, 3, axis=1), np.repeat(doh, 3, axis=1)
    k, v = _rand((1, 1, 30, 8), 70), _rand((1, 1, 30, 8), 71)
    o, _ = oracle.fwd_gqa(q, k, v, 0.35, True)
    assert np.array_equal(o[:, 0], o[:, 1]) and np.array_equal(o[:, 0], o[:, 2])
    _, dk, dv, _ = oracle.bwd_gqa(q, k, v, do, 0.35, True)
    _, dk1, dv1, _ = oracle.bwd(qh, k, v, doh, 0.35, True)
    np.testing.assert_allclose(dv, 3 * dv1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk, 3 * dk1, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------------------------
# Mask and shape variants (§4.5 sliding window, §4.2 cross-attention)
# --------------------------------------------------------------------------------------------
def _torch_masked(q, k, v, do, scale, wl, wr):
    Q, K, V = (torch.from_numpy(x.astype(np.float64)).requires_grad_() for x in (q, k, v))
    nq, nk = q.shape[2], k.shape[2]
    i = torch.arange(nq)[:, None] + (nk - nq)
    j = torch.arange(nk)[None, :]
    vis = torch.ones(nq, nk, dtype=torch.bool)
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    S = (Q @ K.transpose(-1, -2) * scale).masked_fill(~vis, float("-inf"))
    rows = vis.any(-1)
    P = torch.softmax(S.masked_fill(~rows[:, None], 0.0), -1) * rows[:, None]
    O = P @ V
    O.backward(torch.from_numpy(do.astype(np.float64)))
    lse = torch.logsumexp(S, -1)
    return O.detach().numpy(), lse.detach().numpy(), Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def test_ex_reduces_to_causal_and_full_bitwise():
    q, k, v, do = (_rand((1, 2, 70, 16), s) for s in (80, 81, 82, 83))
    for causal, (wl, wr) in ((True, (-1, 0)), (False, (-1, -1))):
        o, lse = oracle.fwd(q, k, v, 0.2, causal)
        oe, lsee = oracle.fwd_ex(q, k, v, 0.2, wl, wr)
        assert np.array_equal(o, oe) and np.array_equal(lse, lsee)
        rq, rk, rv, _ = oracle.bwd(q, k, v, do, 0.2, causal)
        eq, ek, ev = oracle.bwd_ex(q, k, v, do, 0.2, wl, wr)
        np.testing.assert_allclose(eq, rq, rtol=0, atol=1e-13)
        np.testing.assert_allclose(ek, rk, rtol=0, atol=1e-13)
        np.testing.assert_allclose(ev, rv, rtol=0, atol=1e-13)


@pytest.mark.parametrize("nq,nk,wl,wr", [(40, 40, 5, 5), (40, 40, 7, 0), (30, 50, -1, -1),
                                         (50, 30, -1, 0), (30, 50, 4, 2), (45, 20, 3, 0)])
def test_ex_matches_torch_with_explicit_mask(nq, nk, wl, wr):
    q, do = _rand((1, 2, nq, 8), 84), _rand((1, 2, nq, 8), 85)
    k, v = _rand((1, 2, nk, 8), 86), _rand((1, 2, nk, 8), 87)
    o, lse = oracle.fwd_ex(q, k, v, 0.3, wl, wr)
    dq, dk, dv = oracle.bwd_ex(q, k, v, do, 0.3, wl, wr)
    ro, rlse, rq, rk, rv = _torch_masked(q, k, v, do, 0.3, wl, wr)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(rlse))
    fin = np.isfinite(rlse)
    np.testing.assert_allclose(lse[fin], rlse[fin], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dq, rq, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, rk, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, rv, rtol=0, atol=1e-12)


def test_zero_window_returns_own_value_and_empty_rows_are_zero():
    q, k, v = (_rand((1, 1, 20, 8), s) for s in (88, 89, 90))
    o, lse = oracle.fwd_ex(q, k, v, 0.5, 0, 0)          # each query sees only its own key
    np.testing.assert_array_equal(o, v.astype(np.float64))
    np.testing.assert_allclose(lse, 0.5 * (q.astype(np.float64) * k).sum(-1), rtol=0, atol=1e-14)
    # 20 queries on 8 keys, bottom-right aligned causal: the first 12 queries see nothing
    q2 = _rand((1, 1, 20, 8), 91)
    o2, lse2 = oracle.fwd_ex(q2, k[:, :, :8], v[:, :, :8], 0.5, -1, 0)
    assert np.all(o2[0, 0, :12] == 0) and np.all(np.isneginf(lse2[0, 0, :12]))
    assert np.all(np.isfinite(lse2[0, 0, 12:]))
