"""Pins for the oracle: checks against things other than the oracle itself.

The oracle (``oracle/oracle.c``) writes out the definition softmax(Q K^T * scale) V from
FlashAttention (DE), "Problematik der Standard-Attention".  These tests tie it to:

1. Q = 0: every visible key gets the same weight, so O_i is the mean of the visible V rows
   and lse_i = ln |J_i| exactly.
2. A dominant key: O_i approaches that key's V row within (|J_i| - 1) e^-gap * 2 max|v|.
3. Every probability row sums to 1 and is zero on masked keys.
4. The blocked online softmax (running max and running sum of exponentials, rescaled per
   block: FlashAttention (DE), "Online-Softmax-Berechnung") gives the two-pass result.
5. Central finite differences of L = sum(O * dO) match dQ, dK, dV.
6. Closed forms and invariances (N = 1, N = 2 sigmoid, key shift, key/value permutation,
   linearity in V) and the hand-evaluated fixtures in ``golden/closed_forms.json``.
7. torch's own float64 scaled_dot_product_attention with autograd, and the separately
   written numpy twin.

A plausible slip in the oracle (a dropped scale, a sign in dS, a transposed operand, a
missed mask term, an off-by-one in the causal rule) breaks at least one of them; the
mutation tests at the end plant such slips in a copy of the oracle's arithmetic (the numpy
twin) and check that the pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import twin

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def bf16_head(N, d, seed, std=1.0):
    """Random bf16-representable values as fp64 arrays (the oracle's input domain)."""
    g = torch.Generator().manual_seed(seed)
    t = (torch.randn((N, d), generator=g) * std).to(torch.bfloat16)
    return t.double().numpy()


def visible(i, j, L, causal):
    return j < L and (not causal or j <= i)


MASKS = [(False, None), (True, None), (False, 5), (True, 7), (True, 1)]


# ---------------------------------------------------------------- pin 1: Q = 0
@pytest.mark.parametrize("causal,L", MASKS)
def test_zero_query_gives_mean_of_visible_values(causal, L):
    N, d = 24, 8
    q = np.zeros((N, d))
    k = bf16_head(N, d, 1)
    v = bf16_head(N, d, 2)
    Lr = N if L is None else L
    O, lse = oracle.head_fwd(q, k, v, 0.3, causal, Lr)
    for i in range(N):
        J = [j for j in range(N) if visible(i, j, Lr, causal)]
        np.testing.assert_allclose(O[i], v[J].mean(axis=0), rtol=0, atol=1e-14)
        assert abs(lse[i] - math.log(len(J))) <= 1e-15
    if causal:
        np.testing.assert_array_equal(O[0], v[0])


# ---------------------------------------------------------------- pin 2: dominant key
@pytest.mark.parametrize("causal", [False, True])
def test_dominant_key_returns_its_value_row(causal):
    N, d = 32, 16
    q = bf16_head(N, d, 3)
    k = bf16_head(N, d, 4)
    v = bf16_head(N, d, 5)
    i, jstar = 20, 6
    k[jstar] = 6.0 * q[i] / np.linalg.norm(q[i]) * math.sqrt(d)
    scale = 1.0 / math.sqrt(d)
    O, _ = oracle.head_fwd(q, k, v, scale, causal, N)
    J = [j for j in range(N) if visible(i, j, N, causal)]
    s = np.array([scale * q[i] @ k[j] for j in J])
    top = s[J.index(jstar)]
    gap = top - max(s[n] for n, j in enumerate(J) if j != jstar)
    assert gap > 20.0
    bound = (len(J) - 1) * math.exp(-gap) * 2 * np.abs(v).max()
    err = np.abs(O[i] - v[jstar]).max()
    assert err <= bound
    assert err <= 1e-6


# ---------------------------------------------------------------- pin 3: row sums
@pytest.mark.parametrize("causal,L", MASKS)
def test_probability_rows_sum_to_one_and_vanish_on_masked_keys(causal, L):
    N, d = 40, 16
    q, k = bf16_head(N, d, 6), bf16_head(N, d, 7)
    Lr = N if L is None else L
    P = oracle.head_probs(q, k, 0.25, causal, Lr)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    for i in range(N):
        for j in range(N):
            if not visible(i, j, Lr, causal):
                assert P[i, j] == 0.0
            else:
                assert P[i, j] > 0.0


# ---------------------------------------------------------------- pin 4: blocked online softmax
def online_blocked_forward(q, k, v, scale, causal, L, block):
    """Test-only fp64 re-derivation of the tiled online softmax.

    Keys are visited block by block; each row keeps its running maximum m and running sum
    l of exponentials and rescales the partial output whenever m grows (FlashAttention (DE),
    "Online-Softmax-Berechnung": the two intermediate values updated per block).
    """
    N, d = q.shape
    O = np.zeros((N, d))
    lse = np.full(N, -np.inf)
    for i in range(N):
        m, l, acc = -np.inf, 0.0, np.zeros(d)
        for j0 in range(0, N, block):
            js = [j for j in range(j0, min(j0 + block, N)) if visible(i, j, L, causal)]
            if not js:
                continue
            s = np.array([scale * q[i] @ k[j] for j in js])
            m_new = max(m, s.max())
            alpha = math.exp(m - m_new) if m > -np.inf else 0.0
            p = np.exp(s - m_new)
            l = alpha * l + p.sum()
            acc = alpha * acc + p @ v[js]
            m = m_new
        if l > 0:
            O[i] = acc / l
            lse[i] = m + math.log(l)
    return O, lse


@pytest.mark.parametrize("block", [1, 3, 16])
@pytest.mark.parametrize("causal,L", MASKS)
def test_blocked_online_softmax_equals_two_pass(block, causal, L):
    N, d = 48, 8
    q, k, v = bf16_head(N, d, 8, 2.0), bf16_head(N, d, 9, 2.0), bf16_head(N, d, 10)
    Lr = N if L is None else L
    O, lse = oracle.head_fwd(q, k, v, 0.5, causal, Lr)
    O2, lse2 = online_blocked_forward(q, k, v, 0.5, causal, Lr, block)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- pin 5: finite differences
@pytest.mark.parametrize("causal,L", [(False, None), (True, None), (False, 7), (True, 9)])
def test_gradients_match_central_differences(causal, L):
    N, d = 12, 6
    q, k, v, do = (bf16_head(N, d, s) for s in (11, 12, 13, 14))
    Lr = N if L is None else L
    scale = 0.7
    g = oracle.head_bwd(q, k, v, do, scale, causal, Lr)
    h = 1e-6

    def loss(q_, k_, v_):
        O, _ = oracle.head_fwd(q_, k_, v_, scale, causal, Lr)
        return float((O * do).sum())

    for name, arr, grad in (("q", q, g["dq"]), ("k", k, g["dk"]), ("v", v, g["dv"])):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = plus, minus
            fd[idx] = (loss(**{f"{n}_": a for n, a in args_p.items()})
                       - loss(**{f"{n}_": a for n, a in args_m.items()})) / (2 * h)
        ref = max(1.0, np.abs(grad).max())
        assert np.abs(fd - grad).max() <= 1e-6 * ref, name


# ---------------------------------------------------------------- pin 6: closed forms
def test_single_token_returns_its_value_and_score():
    q, k, v = bf16_head(1, 8, 15), bf16_head(1, 8, 16), bf16_head(1, 8, 17)
    O, lse = oracle.head_fwd(q, k, v, 0.125, False, 1)
    np.testing.assert_array_equal(O[0], v[0])
    assert abs(lse[0] - 0.125 * float(q[0] @ k[0])) <= 1e-15


def test_two_keys_give_a_sigmoid():
    q, k, v = bf16_head(2, 8, 18), bf16_head(2, 8, 19), bf16_head(2, 8, 20)
    P = oracle.head_probs(q, k, 0.4, False, 2)
    for i in range(2):
        s0, s1 = 0.4 * q[i] @ k[0], 0.4 * q[i] @ k[1]
        assert abs(P[i, 0] - 1.0 / (1.0 + math.exp(-(s0 - s1)))) <= 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_shifting_every_key_leaves_O_and_moves_lse(causal):
    N, d = 20, 8
    q, k, v = bf16_head(N, d, 21), bf16_head(N, d, 22), bf16_head(N, d, 23)
    c = bf16_head(1, d, 24)[0]
    O, lse = oracle.head_fwd(q, k, v, 0.3, causal, N)
    O2, lse2 = oracle.head_fwd(q, k + c, v, 0.3, causal, N)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse + 0.3 * q @ c, rtol=0, atol=1e-12)


def test_permuting_keys_and_values_leaves_O():
    N, d = 20, 8
    q, k, v = bf16_head(N, d, 25), bf16_head(N, d, 26), bf16_head(N, d, 27)
    perm = np.random.default_rng(0).permutation(N)
    O, lse = oracle.head_fwd(q, k, v, 0.3, False, N)
    O2, lse2 = oracle.head_fwd(q, k[perm], v[perm], 0.3, False, N)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal,L", MASKS)
def test_output_is_linear_in_V(causal, L):
    N, d = 20, 8
    q, k = bf16_head(N, d, 28), bf16_head(N, d, 29)
    v1, v2 = bf16_head(N, d, 30), bf16_head(N, d, 31)
    Lr = N if L is None else L
    O1, _ = oracle.head_fwd(q, k, v1, 0.3, causal, Lr)
    O2, _ = oracle.head_fwd(q, k, v2, 0.3, causal, Lr)
    O3, _ = oracle.head_fwd(q, k, 2.0 * v1 - 3.0 * v2, 0.3, causal, Lr)
    np.testing.assert_allclose(O3, 2.0 * O1 - 3.0 * O2, rtol=0, atol=1e-12)


def _eval(expr):
    env = {"__builtins__": {}, "e": math.e, "exp": math.exp, "log": math.log,
           "sigmoid": lambda x: 1.0 / (1.0 + math.exp(-x))}
    return float(eval(expr, env))  # expressions come from the committed fixture only


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_evaluated_fixtures(case):
    q, k, v = (np.array(case[n], dtype=np.float64) for n in ("q", "k", "v"))
    O, lse = oracle.head_fwd(q, k, v, case["scale"], case["causal"], case["L"])
    np.testing.assert_allclose(O, [[_eval(x) for x in r] for r in case["O"]], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, [_eval(x) for x in case["lse"]], rtol=0, atol=1e-15)
    if "dO" in case:
        g = oracle.head_bwd(q, k, v, np.array(case["dO"], dtype=np.float64), case["scale"],
                            case["causal"], case["L"])
        for name, key in (("dQ", "dq"), ("dK", "dk"), ("dV", "dv")):
            np.testing.assert_allclose(g[key], [[_eval(x) for x in r] for r in case[name]],
                                       rtol=0, atol=1e-15)


# ---------------------------------------------------------------- pin 7: torch fp64 + numpy twin
def torch_reference(q, k, v, do, scale, causal, L):
    N = q.shape[0]
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    mask = j < L
    if causal:
        mask = mask & (j <= i)
    O = torch.nn.functional.scaled_dot_product_attention(
        tq[None, None], tk[None, None], tv[None, None], attn_mask=mask[None, None], scale=scale)[0, 0]
    O.backward(torch.tensor(do, dtype=torch.float64))
    return O.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("causal,L", MASKS)
def test_matches_torch_float64_attention_and_autograd(causal, L):
    N, d = 33, 16
    q, k, v, do = (bf16_head(N, d, s) for s in (32, 33, 34, 35))
    Lr = N if L is None else L
    g = oracle.head_bwd(q, k, v, do, 0.25, causal, Lr)
    O, dq, dk, dv = torch_reference(q, k, v, do, 0.25, causal, Lr)
    for a, b in ((g["o"], O), (g["dq"], dq), (g["dk"], dk), (g["dv"], dv)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,L", MASKS)
def test_matches_numpy_twin(causal, L):
    N, d = 40, 32
    q, k, v, do = (bf16_head(N, d, s) for s in (36, 37, 38, 39))
    Lr = N if L is None else L
    g = oracle.head_bwd(q, k, v, do, 0.2, causal, Lr)
    t = twin.backward(q, k, v, do, 0.2, causal, Lr)
    for name in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(g[name], t[name], rtol=0, atol=1e-12, err_msg=name)


# ---------------------------------------------------------------- wrappers agree with each other
def test_row_subsets_and_batched_wrappers_agree_with_full_heads():
    B, H, N, d = 2, 2, 24, 8
    g = torch.Generator().manual_seed(40)
    q, k, v, do = ((torch.randn((B, H, N, d), generator=g)).to(torch.bfloat16) for _ in range(4))
    seqlens = torch.tensor([24, 9], dtype=torch.int32)
    O, lse = oracle.attention_fwd(q, k, v, 0.3, True, seqlens)
    full = oracle.attention_bwd(q, k, v, do, 0.3, True, seqlens)
    np.testing.assert_array_equal(full["o"], O)
    for b in range(B):
        for h in range(H):
            L = int(seqlens[b])
            rows = [0, 5, 8, 9, 23]
            Or, lser = oracle.head_fwd_rows(q[b, h], k[b, h], v[b, h], rows, 0.3, True, L)
            np.testing.assert_array_equal(Or, O[b, h, rows])
            np.testing.assert_array_equal(lser, lse[b, h, rows])
            r = oracle.head_bwd_rows(q[b, h], k[b, h], v[b, h], do[b, h], rows, [1, 8, 20],
                                     0.3, True, L)
            np.testing.assert_allclose(r["dq"], full["dq"][b, h, rows], rtol=0, atol=1e-15)
            np.testing.assert_allclose(r["dk"], full["dk"][b, h, [1, 8, 20]], rtol=0, atol=1e-15)
            np.testing.assert_allclose(r["dv"], full["dv"][b, h, [1, 8, 20]], rtol=0, atol=1e-15)
    # padded keys (j >= L) receive no gradient
    assert np.all(full["dk"][1, :, 9:] == 0) and np.all(full["dv"][1, :, 9:] == 0)


def test_rejects_bad_arguments():
    q = np.zeros((4, 2))
    with pytest.raises(RuntimeError):
        oracle.head_fwd(q, q, q, 1.0, False, 5)
    with pytest.raises(RuntimeError):
        oracle.head_fwd_rows(q, q, q, [4], 1.0, False, 4)


# ---------------------------------------------------------------- the pins catch planted slips
def _mutant(kind):
    """A copy of the twin's arithmetic with one plausible slip planted in it (CPU only)."""

    def fwd_bwd(q, k, v, do, scale, causal, L):
        N = q.shape[0]
        vis = twin.visible_mask(N, causal, L)
        if kind == "causal-off-by-one":
            vis = twin.visible_mask(N, False, L) & (np.arange(N)[None, :] < np.arange(N)[:, None])
            vis[0, 0] = True
        S = (q @ k.T) * (1.0 if kind == "dropped-scale" else scale)
        if kind == "transposed-scores":
            S = S.T
        S = np.where(vis, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        P = E / E.sum(axis=1, keepdims=True)
        O = P @ v
        dP = do @ v.T
        D = (do * O).sum(axis=1, keepdims=True)
        dS = P * (dP + D) if kind == "dS-sign" else P * (dP - D)
        dq = scale * dS @ k
        dk = scale * dS.T @ q
        dv = P @ do if kind == "dV-untransposed" else P.T @ do
        return {"o": O, "dq": dq, "dk": dk, "dv": dv}

    return fwd_bwd


@pytest.mark.parametrize("kind", ["dropped-scale", "transposed-scores", "dS-sign",
                                  "dV-untransposed", "causal-off-by-one"])
def test_pins_catch_planted_slips(kind):
    """Each slip, planted in a CPU copy of the arithmetic, is caught by the torch pin."""
    N, d = 16, 8
    q, k, v, do = (bf16_head(N, d, s) for s in (41, 42, 43, 44))
    causal = kind == "causal-off-by-one"
    got = _mutant(kind)(q, k, v, do, 0.3, causal, N)
    O, dq, dk, dv = torch_reference(q, k, v, do, 0.3, causal, N)
    worst = max(np.abs(got[n] - r).max() for n, r in (("o", O), ("dq", dq), ("dk", dk), ("dv", dv)))
    assert worst > 1e-6


# ---------------------------------------------------------------- grouped-query attention
def test_gqa_with_one_query_head_per_kv_head_is_plain_attention():
    g = torch.Generator().manual_seed(50)
    q, k, v, do = ((torch.randn((2, 3, 20, 8), generator=g)).to(torch.bfloat16) for _ in range(4))
    a = oracle.attention_bwd_gqa(q, k, v, do, 0.3, True, [20, 11])
    b = oracle.attention_bwd(q, k, v, do, 0.3, True, [20, 11])
    for n in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_array_equal(a[n], b[n])


@pytest.mark.parametrize("H,H_kv,causal", [(4, 2, False), (3, 1, True)])
def test_gqa_gradients_match_central_differences(H, H_kv, causal):
    """A shared key/value element feeds several query heads: its gradient is their sum."""
    N, d = 6, 4
    g = torch.Generator().manual_seed(51 + H)
    q = torch.randn((1, H, N, d), generator=g).to(torch.bfloat16).double().numpy()
    k = torch.randn((1, H_kv, N, d), generator=g).to(torch.bfloat16).double().numpy()
    v = torch.randn((1, H_kv, N, d), generator=g).to(torch.bfloat16).double().numpy()
    do = torch.randn((1, H, N, d), generator=g).to(torch.bfloat16).double().numpy()
    grads = oracle.attention_bwd_gqa(q, k, v, do, 0.6, causal)
    h = 1e-6

    def loss(q_, k_, v_):
        O, _ = oracle.attention_fwd_gqa(q_, k_, v_, 0.6, causal)
        return float((O * do).sum())

    for name, arr, grad in (("q", q, grads["dq"]), ("k", k, grads["dk"]), ("v", v, grads["dv"])):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][idx] += h
            lp = loss(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * h
            lm = loss(args["q"], args["k"], args["v"])
            fd[idx] = (lp - lm) / (2 * h)
        assert np.abs(fd - grad).max() <= 1e-6 * max(1.0, np.abs(grad).max()), name


# ------------------------------------------------------------------ packed variable-length
CU_PACK = [0, 3, 3, 8, 9, 13]   # lengths 3, 0 (empty), 5, 1, 4; rows 13..14 belong to no sequence


def _packed(T, H, H_kv, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((T, H, d), generator=g).to(torch.bfloat16).double().numpy()
    k = torch.randn((T, H_kv, d), generator=g).to(torch.bfloat16).double().numpy()
    v = torch.randn((T, H_kv, d), generator=g).to(torch.bfloat16).double().numpy()
    do = torch.randn((T, H, d), generator=g).to(torch.bfloat16).double().numpy()
    return q, k, v, do


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_zero_query_gives_each_sequences_own_running_mean(causal):
    """Q = 0: row i of a sequence averages the value rows of ITS sequence that it sees (all of
    them, or its first i + 1 when causal), and lse = ln(count) exactly.  A slice boundary off
    by one, or a sequence leaking into the next, changes the mean."""
    T, H, H_kv, d = 15, 4, 2, 3
    _, k, v, _ = _packed(T, H, H_kv, d, 61)
    q = np.zeros((T, H, d))
    O, lse = oracle.attention_fwd_varlen(q, k, v, np.array(CU_PACK), 0.7, causal)
    for t0, t1 in zip(CU_PACK[:-1], CU_PACK[1:]):
        for i in range(t1 - t0):
            n = (i + 1) if causal else (t1 - t0)
            for h in range(H):
                want = v[t0:t0 + n, h // 2].mean(axis=0)
                assert np.abs(O[t0 + i, h] - want).max() < 1e-15
                assert lse[h, t0 + i] == math.log(n)
    assert np.all(O[13:] == 0) and np.all(np.isnan(lse[:, 13:]))


def test_varlen_sequences_are_independent():
    """Changing every input row of one sequence leaves every other sequence's outputs as they
    were, bit for bit."""
    T, H, H_kv, d = 15, 2, 1, 4
    q, k, v, _ = _packed(T, H, H_kv, d, 62)
    O1, l1 = oracle.attention_fwd_varlen(q, k, v, np.array(CU_PACK), 0.5, True)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[3:8] += 1.0
    k2[3:8] -= 2.0
    v2[3:8] *= 3.0
    O2, l2 = oracle.attention_fwd_varlen(q2, k2, v2, np.array(CU_PACK), 0.5, True)
    other = np.r_[0:3, 8:13]
    assert np.array_equal(O1[other], O2[other]) and np.array_equal(l1[:, other], l2[:, other])
    assert not np.allclose(O1[3:8], O2[3:8])


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_gradients_match_central_differences(causal):
    """Gradients on the packed layout (scatter of per-sequence, per-head pieces) against central
    differences of the packed forward."""
    cu = np.array([0, 2, 2, 5, 6])
    T, H, H_kv, d = 7, 2, 1, 3
    q, k, v, do = _packed(T, H, H_kv, d, 63)
    grads = oracle.attention_bwd_varlen(q, k, v, do, cu, 0.8, causal)
    h = 1e-6

    def loss(q_, k_, v_):
        O, _ = oracle.attention_fwd_varlen(q_, k_, v_, cu, 0.8, causal)
        return float((O * do).sum())

    for name, arr, grad in (("q", q, grads["dq"]), ("k", k, grads["dk"]), ("v", v, grads["dv"])):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][idx] += h
            lp = loss(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * h
            lm = loss(args["q"], args["k"], args["v"])
            fd[idx] = (lp - lm) / (2 * h)
        assert np.abs(fd - grad).max() <= 1e-6 * max(1.0, np.abs(grad).max()), name
    assert np.all(grads["dq"][6] == 0) and np.all(grads["dk"][6] == 0)


def test_varlen_rejects_offsets_outside_the_pack():
    q, k, v, _ = _packed(5, 1, 1, 2, 64)
    for cu in ([0, 3, 2], [0, 6], [-1, 2]):
        with pytest.raises(ValueError):
            oracle.attention_fwd_varlen(q, k, v, np.array(cu), 1.0, False)


# ------------------------------------------------------------------ decode (KV cache)
def _decode_inputs(B, H, H_kv, Nq, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16).double().numpy()
    k = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16).double().numpy()
    v = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16).double().numpy()
    return q, k, v


def test_decode_with_all_positions_as_queries_is_causal_self_attention():
    """Nq = L: the end-aligned causal mask becomes the ordinary j <= i mask, so the decode
    definition must equal the pinned C oracle's causal self-attention on the same rows."""
    q, k, v = _decode_inputs(1, 2, 2, 9, 9, 5, 71)
    O, lse = oracle.attention_decode(q, k, v, 0.4, True)
    for h in range(2):
        O_ref, lse_ref = oracle.head_fwd(q[0, h], k[0, h], v[0, h], 0.4, True)
        assert np.abs(O[0, h] - O_ref).max() < 1e-13
        assert np.abs(lse[0, h] - lse_ref).max() < 1e-13


def test_decode_zero_queries_average_the_visible_end_aligned_cache_rows():
    """Q = 0: query i averages value rows 0 .. lim-1 with lim = L - Nq + i + 1 (causal) or L,
    lse = ln(lim) exactly; cache rows >= L never enter; a query seeing nothing gets (0, -inf)."""
    B, H, H_kv, Nq, N, d = 2, 4, 2, 3, 12, 3
    _, k, v = _decode_inputs(B, H, H_kv, Nq, N, d, 72)
    q = np.zeros((B, H, Nq, d))
    lens = [7, 2]
    for causal in (False, True):
        O, lse = oracle.attention_decode(q, k, v, 1.3, causal, lens)
        for b in range(B):
            L = lens[b]
            for h in range(H):
                for i in range(Nq):
                    lim = min(L, L - Nq + i + 1) if causal else L
                    if lim <= 0:
                        assert np.all(O[b, h, i] == 0) and lse[b, h, i] == -np.inf
                        continue
                    assert np.abs(O[b, h, i] - v[b, h // 2, :lim].mean(axis=0)).max() < 1e-15
                    assert lse[b, h, i] == math.log(lim)


def test_decode_merging_key_ranges_by_lse_gives_the_whole_result():
    """The split-KV identity the GPU combine relies on, checked on the definition: attention
    over the cache rows [0, a) and [a, L) separately, merged by lse = log(e^lse1 + e^lse2) and
    O = e^(lse1 - lse) O1 + e^(lse2 - lse) O2, equals attention over [0, L)."""
    q, k, v = _decode_inputs(1, 2, 1, 2, 20, 4, 73)
    O, lse = oracle.attention_decode(q, k, v, 0.5, False)
    a = 7
    O1, l1 = oracle.attention_decode(q, k[:, :, :a], v[:, :, :a], 0.5, False)
    O2, l2 = oracle.attention_decode(q, k[:, :, a:], v[:, :, a:], 0.5, False)
    lm = np.logaddexp(l1, l2)
    Om = np.exp(l1 - lm)[..., None] * O1 + np.exp(l2 - lm)[..., None] * O2
    assert np.abs(lm - lse).max() < 1e-13 and np.abs(Om - O).max() < 1e-13


def test_decode_single_query_causal_equals_non_causal_and_torch():
    """Nq = 1 sees the whole valid cache with or without the causal flag; both agree with
    torch float64 scaled_dot_product_attention on the valid rows."""
    q, k, v = _decode_inputs(2, 4, 1, 1, 10, 6, 74)
    lens = [10, 4]
    Oc, lc = oracle.attention_decode(q, k, v, 0.3, True, lens)
    On, ln_ = oracle.attention_decode(q, k, v, 0.3, False, lens)
    assert np.array_equal(Oc, On) and np.array_equal(lc, ln_)
    for b in range(2):
        L = lens[b]
        for h in range(4):
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, h][None]), torch.from_numpy(k[b, 0, :L][None]),
                torch.from_numpy(v[b, 0, :L][None]), scale=0.3)[0]
            assert np.abs(On[b, h] - ref.numpy()).max() < 1e-12


# ------------------------------------------------------------------ FP8 (e4m3) inputs
def test_e4m3_decoding_follows_the_bit_fields():
    """Hand-decoded codes: 0x38 = 2^0 = 1, 0x7E = 1.75 * 2^8 = 448 (largest finite),
    0x01 = 2^-9 (smallest subnormal), 0x08 = 2^-6 (smallest normal), 0x07 = 7/8 * 2^-6,
    0xC5 = -(1 + 5/8) * 2 = -3.25, 0x7F = NaN."""
    codes = np.array([0x38, 0x7E, 0x01, 0x08, 0x07, 0xC5, 0x7F, 0x00, 0x80])
    got = oracle.decode_e4m3(codes)
    want = [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, 7 / 8 * 2.0 ** -6, -3.25, np.nan, 0.0, -0.0]
    np.testing.assert_array_equal(got, np.array(want))


def test_e4m3_decoding_agrees_with_torch_on_every_finite_code():
    """All 254 finite codes against torch's float8_e4m3fn -> float64 conversion."""
    codes = torch.arange(256, dtype=torch.uint8)
    mine = oracle.decode_e4m3(codes.numpy())
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(ref)
    assert finite.sum() == 254
    np.testing.assert_array_equal(mine[finite], ref[finite])
    assert np.isnan(mine[~finite]).all()


def test_fp8_attention_is_attention_of_the_dequantised_values():
    """Scaling a head's descale by 2 and halving its codes' values is the same input; the FP8
    oracle must see only code * descale (K descale folded into scores, V into O)."""
    import workloads
    w = workloads.custom(1, 2, 20, 8, True, seed=81)
    f = workloads.make_fp8_inputs(w)
    O, lse = oracle.attention_fwd_fp8(f.q, f.k, f.v, f.q_descale, f.k_descale, f.v_descale,
                                      0.35, True)
    q = oracle.decode_e4m3(f.q) * f.q_descale.double().numpy()[:, :, None, None]
    k = oracle.decode_e4m3(f.k) * f.k_descale.double().numpy()[:, :, None, None]
    v = oracle.decode_e4m3(f.v) * f.v_descale.double().numpy()[:, :, None, None]
    O2, lse2 = oracle.attention_fwd_gqa(q, k, 2.0 * v, 0.35, True)
    assert np.abs(2.0 * O - O2).max() < 1e-12 and np.abs(lse - lse2).max() == 0.0
    # the quantised values stay within one e4m3 step (2^-3 relative) of the fp32 draws
    assert np.all(np.abs(f.q.float().abs().numpy()) <= 448.0)


# ---------------------------------------------------------------- dQ rounding magnitudes
@pytest.mark.parametrize("causal", [False, True])
def test_dq_magnitude_sums_bound_dq_and_match_brute_force(causal):
    """oracle.dq_magnitude_sums (used by the tolerances of the fixed-point dQ tests): checked
    against explicit loops over keys written here from the definitions (softmax of the scaled
    scores over the visible keys, dS = P (dP - D), D = dO . O), against the C oracle's dQ
    (|dQ_il| <= scale * sum_j |dS_ij| |k_jl|, the triangle inequality), and on special cases
    (one visible key: dS = 0, so the first sum vanishes; Q = 0: P is uniform, so the second
    sum is |dO| |O| times the mean of |k|)."""
    N, d, scale = 9, 4, 0.37
    q, k, v, do = (bf16_head(N, d, 900 + i) for i in range(4))
    rows = [0, 3, 8]
    got = oracle.dq_magnitude_sums(q, k, v, do, rows, scale, causal)
    for r, i in enumerate(rows):
        J = [j for j in range(N) if visible(i, j, N, causal)]
        s = [scale * sum(q[i, c] * k[j, c] for c in range(d)) for j in J]
        m = max(s)
        z = sum(math.exp(x - m) for x in s)
        P = [math.exp(x - m) / z for x in s]
        O = [sum(P[t] * v[j, c] for t, j in enumerate(J)) for c in range(d)]
        D = sum(do[i, c] * O[c] for c in range(d))
        dS = [P[t] * (sum(do[i, c] * v[j, c] for c in range(d)) - D) for t, j in enumerate(J)]
        no = math.sqrt(sum(x * x for x in do[i])) * math.sqrt(sum(x * x for x in O))
        for c in range(d):
            a = sum(abs(dS[t]) * abs(k[j, c]) for t, j in enumerate(J))
            b = no * sum(P[t] * abs(k[j, c]) for t, j in enumerate(J))
            assert abs(got["abs_dS_k"][r, c] - a) <= 1e-12 * max(1.0, a)
            assert abs(got["D_term"][r, c] - b) <= 1e-12 * max(1.0, b)
    ref = oracle.head_bwd(q, k, v, do, scale, causal)
    bound = oracle.dq_magnitude_sums(q, k, v, do, list(range(N)), scale, causal)
    assert np.all(np.abs(ref["dq"]) <= scale * bound["abs_dS_k"] * (1 + 1e-12) + 1e-15)
    if causal:
        assert np.all(bound["abs_dS_k"][0] == 0)  # row 0 sees one key
    z = oracle.dq_magnitude_sums(np.zeros_like(q), k, v, do, [N - 1], scale, False)
    O = v.mean(0)
    want = np.linalg.norm(do[N - 1]) * np.linalg.norm(O) * np.abs(k).mean(0)
    assert np.allclose(z["D_term"][0], want, rtol=1e-12, atol=0)
