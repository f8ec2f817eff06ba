"""Pins of the FP64 oracle against facts that do not come from the oracle itself.

Each test names what pins it: a hand-worked example (tests/golden), a library
routine, a closed form, an invariant of the mathematics, brute force on tiny inputs,
or an independent algebraic form of the same recurrence (tests/kda_forms.py).
"""
import json
import math
import os

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st
import pytest
import scipy.special
import torch

import oracle
from synth import core_inputs
from tests.kda_forms import brute_force, chunked_lookahead, chunked_wy

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_head(T, D, seed, g_scale=1.0, s0_std=0.3):
    r = _rng(seed)
    q = _unit(r.standard_normal((T, D)))
    k = _unit(r.standard_normal((T, D)))
    v = r.standard_normal((T, D))
    g = -g_scale * np.log1p(np.exp(r.standard_normal((T, D))))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal(T)))
    s0 = s0_std * r.standard_normal((D, D))
    return q, k, v, g, beta, s0


def _oracle_head(q, k, v, g, beta, s0, scale=1.0):
    o, S = oracle.recurrence(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                             beta[None, :, None], s0[None, None], scale)
    return o[0, :, 0], S[0, 0]


# ---------------------------------------------------------------- hand-worked example

def test_hand_worked_two_tokens():
    """Pinned by tests/golden/hand_worked_d2.json (worked by hand, exact decimals)."""
    with open(os.path.join(GOLDEN, "hand_worked_d2.json")) as f:
        G = json.load(f)
    g = np.log(np.array(G["exp_g"]))
    o, S = _oracle_head(np.array(G["q"]), np.array(G["k"]), np.array(G["v"]), g,
                        np.array(G["beta"]), np.array(G["S0"]), G["scale"])
    np.testing.assert_allclose(o, np.array(G["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S, np.array(G["S_T"]), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- BF16 rounding

def test_bf16_round_matches_library_conversion():
    """Pinned by torch's float32 -> bfloat16 conversion (RNE) on float32-exact inputs,
    including ties, subnormals, the overflow boundary and signed zeros."""
    r = _rng(1)
    vals = [0.0, -0.0, 1.0, -1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, 1.5 + 2 ** -8,
            2 ** -126, 2 ** -130, 3 * 2 ** -134, 2 ** -133, 2 ** -134, 3.3895313892515355e38,
            3.3961e38, 3.4e38, -3.4e38, 65504.0, 1e-40, -1e-41]
    x = np.concatenate([np.array(vals), r.standard_normal(20000) * np.exp(r.uniform(-80, 80, 20000))])
    x32 = x.astype(np.float32)
    expect = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_round(x32.astype(np.float64))
    assert np.array_equal(got, expect) and np.array_equal(np.signbit(got), np.signbit(expect))


# ---------------------------------------------------------------- gate

def test_softplus_sigmoid_against_library():
    """Pinned by numpy logaddexp (log(1+e^x)) and scipy expit (logistic)."""
    x = np.linspace(-700, 700, 20001)
    np.testing.assert_allclose(oracle.softplus(x), np.logaddexp(0.0, x), rtol=1e-15, atol=1e-300)
    np.testing.assert_allclose(oracle.sigmoid(x), scipy.special.expit(x), rtol=1e-15, atol=1e-300)
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), abs=1e-16)


def test_gate_per_head_a_log_per_channel_dt_bias():
    """Indexing pins (Glm5NextKdaWeights: dt_bias per channel, a_log per head): a change
    of a_log[h] moves only head h; a change of dt_bias[c] moves only channel c; g <= 0;
    the special value a_log = 0, g_raw + dt_bias = 0 gives -ln 2."""
    H, D, T = 3, 4, 5
    r = _rng(2)
    g_raw = r.standard_normal((T, H * D))
    dt = r.uniform(-1, 1, H * D)
    al = r.uniform(-1, 1, H)
    g0 = oracle.gate(g_raw, dt, al, H, D)
    assert g0.shape == (T, H, D) and np.all(g0 <= 0)
    al2 = al.copy()
    al2[1] += 0.5
    d = oracle.gate(g_raw, dt, al2, H, D) - g0
    assert np.all(d[:, 1] != 0) and np.all(d[:, [0, 2]] == 0)
    dt2 = dt.copy()
    dt2[2 * D + 3] += 0.5
    d = (oracle.gate(g_raw, dt2, al, H, D) - g0).reshape(T, H * D)
    assert np.all(d[:, 2 * D + 3] != 0) and np.count_nonzero(d) == T
    z = oracle.gate(np.zeros((1, H * D)), np.zeros(H * D), np.zeros(H), H, D)
    np.testing.assert_allclose(z, -math.log(2.0), rtol=1e-15)
    far = oracle.gate(np.full((1, H * D), -800.0), np.zeros(H * D), al, H, D)
    assert np.all(far == 0.0) or np.all(np.abs(far) < 1e-300)
    # large argument: softplus(x) -> x, so g -> -exp(a_log) x
    big = oracle.gate(np.full((1, H * D), 50.0), np.zeros(H * D), al, H, D)
    np.testing.assert_allclose(big[0], -np.exp(al)[:, None] * 50.0 * np.ones((H, D)), rtol=1e-15)


# ---------------------------------------------------------------- recurrence

@pytest.mark.parametrize("T,D,seed", [(1, 1, 0), (3, 2, 1), (6, 3, 2), (8, 4, 3)])
def test_recurrence_brute_force(T, D, seed):
    """Pinned by the explicit product of D x D transition matrices (kda_forms.brute_force)."""
    args = _rand_head(T, D, seed)
    o, S = _oracle_head(*args, scale=0.7)
    ob, Sb = brute_force(*args, scale=0.7)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, Sb, rtol=1e-12, atol=1e-13)


def test_recurrence_beta_zero_closed_form():
    """beta = 0: no update, S_t = diag(exp(sum_{s<=t} g_s)) S0 and o_t = S_t^T q_t."""
    q, k, v, g, beta, s0 = _rand_head(40, 8, 5)
    o, S = _oracle_head(q, k, v, g, np.zeros_like(beta), s0)
    G = np.cumsum(g, axis=0)
    np.testing.assert_allclose(S, np.exp(G[-1])[:, None] * s0, rtol=1e-12, atol=1e-300)
    for t in range(40):
        np.testing.assert_allclose(o[t], (np.exp(G[t])[:, None] * s0).T @ q[t], rtol=1e-11, atol=1e-14)


def test_recurrence_exact_retrieval_orthonormal_keys():
    """g = 0, beta = 1, orthonormal keys, S0 = 0: S_T = sum_j k_j v_j^T, so S_T^T k_j = v_j."""
    D, T = 16, 16
    r = _rng(6)
    Qm, _ = np.linalg.qr(r.standard_normal((D, D)))
    k = Qm.T[:T]
    v = r.standard_normal((T, D))
    q = _unit(r.standard_normal((T, D)))
    _, S = _oracle_head(q, k, v, np.zeros((T, D)), np.ones(T), np.zeros((D, D)))
    np.testing.assert_allclose(k @ S, v, atol=1e-12)


def test_recurrence_scalar_closed_form():
    """D = 1: s_T = s0 prod_t a_t + sum_j beta_j k_j v_j prod_{t>j} a_t, a_t = e^{g_t}(1 - beta_t k_t^2)."""
    T = 30
    r = _rng(7)
    k = r.uniform(-1, 1, T)
    v = r.standard_normal(T)
    g = -r.uniform(0, 0.5, T)
    b = r.uniform(0, 1, T)
    s0 = 0.8
    a = np.exp(g) * (1 - b * k * k)
    expect = s0 * np.prod(a) + sum(b[j] * k[j] * v[j] * np.prod(a[j + 1:]) for j in range(T))
    _, S = _oracle_head(np.ones((T, 1)), k[:, None], v[:, None], g[:, None], b, np.array([[s0]]))
    assert S[0, 0] == pytest.approx(expect, rel=1e-13)


def test_recurrence_per_token_invariant_and_bound():
    """Unit k_t: S_t^T k_t = (1 - beta_t) S'^T k_t + beta_t v_t with S' = diag(e^g_t) S_{t-1};
    and the step is non-expansive: ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t||."""
    q, k, v, g, beta, s0 = _rand_head(50, 12, 8, g_scale=0.2, s0_std=1.0)
    S_prev = s0
    for t in range(50):
        _, S = _oracle_head(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1], S_prev)
        Sp = np.exp(g[t])[:, None] * S_prev
        np.testing.assert_allclose(S.T @ k[t], (1 - beta[t]) * (Sp.T @ k[t]) + beta[t] * v[t],
                                   rtol=1e-12, atol=1e-12)
        assert np.linalg.norm(S) <= np.linalg.norm(S_prev) + beta[t] * np.linalg.norm(v[t]) + 1e-12
        S_prev = S


@pytest.mark.parametrize("T,D,C,seed", [(64, 64, 64, 0), (200, 32, 64, 1), (130, 128, 64, 2), (37, 8, 16, 3)])
def test_chunked_equals_recurrent(T, D, C, seed):
    """Pinned by the chunked WY/UT form (kda_forms.chunked_wy), which shares no code with the
    token loop: the two must agree to FP64 rounding, including a ragged last chunk."""
    args = _rand_head(T, D, seed, g_scale=1.5)
    o, S = _oracle_head(*args, scale=0.5)
    oc, Sc = chunked_wy(*args, scale=0.5, C=C)
    np.testing.assert_allclose(o, oc, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S, Sc, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("T,D,C,seed", [(200, 32, 64, 4), (130, 16, 16, 5), (64, 8, 64, 6)])
def test_lookahead_chain_equals_chunked_and_recurrent(T, D, C, seed):
    """The U-carried inter-chunk chain (kda_forms.chunked_lookahead: U_{c+1} from U_c through
    Z = W_{c+1} K-bar_c^T, the state one step behind) gives the chunked form's and the token
    recurrence's outputs and final state to FP64 rounding, ragged last chunk included."""
    args = _rand_head(T, D, seed, g_scale=1.5)
    o, S = _oracle_head(*args, scale=0.7)
    ol, Sl = chunked_lookahead(*args, scale=0.7, C=C)
    np.testing.assert_allclose(ol, o, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(Sl, S, rtol=1e-9, atol=1e-11)


@settings(max_examples=25, deadline=None)
@given(T=st.integers(1, 90), D=st.sampled_from([1, 2, 5, 8, 16]), C=st.sampled_from([4, 16, 64]),
       seed=st.integers(0, 2 ** 31 - 1), g_scale=st.floats(0.0, 3.0), scale=st.floats(0.1, 2.0))
def test_three_forms_agree_on_random_shapes(T, D, C, seed, g_scale, scale):
    """Property: for any length (ragged chunks included), head size, chunk size, decay strength
    and read-out scale, the token recurrence (the oracle), the chunked WY/UT form and the
    U-carried chain give the same outputs and final state to FP64 rounding."""
    args = _rand_head(T, D, seed, g_scale=g_scale)
    o, S = _oracle_head(*args, scale=scale)
    for form in (chunked_wy, chunked_lookahead):
        of, Sf = form(*args, scale=scale, C=C)
        np.testing.assert_allclose(of, o, rtol=1e-8, atol=1e-10)
        np.testing.assert_allclose(Sf, S, rtol=1e-8, atol=1e-10)


def test_oracle_uses_heads_and_sequences_independently():
    """Head h's outputs depend only on head h's inputs; sequences are independent; a split
    prefill from the carried state equals the whole prefill (bit for bit: same operations)."""
    ci = core_inputs(2, 48, 3, 16, seed=11, s0_std=0.1)
    g = oracle.gate(ci.g_raw.float(), ci.dt_bias, ci.a_log, 3, 16)
    beta = oracle.sigmoid(ci.b_logit)
    o, S = oracle.recurrence(ci.q, ci.k, ci.v, g, beta, ci.s0)
    o1, S1 = oracle.recurrence(ci.q[:, :20], ci.k[:, :20], ci.v[:, :20], g[:, :20], beta[:, :20], ci.s0)
    o2, S2 = oracle.recurrence(ci.q[:, 20:], ci.k[:, 20:], ci.v[:, 20:], g[:, 20:], beta[:, 20:], S1)
    assert np.array_equal(np.concatenate([o1, o2], axis=1), o) and np.array_equal(S2, S)
    q2 = ci.q.clone()
    q2[1, :, 2] = 0.0
    o3, _ = oracle.recurrence(q2, ci.k, ci.v, g, beta, ci.s0)
    assert np.array_equal(o3[0], o[0]) and np.array_equal(o3[1, :, :2], o[1, :, :2])
    assert np.all(o3[1, :, 2] == 0)


# ---------------------------------------------------------------- front end / back end

def test_conv_against_numpy_convolve():
    """Causal depthwise conv from the carried state, pinned by numpy.convolve per channel;
    SiLU pinned by scipy expit; the new state is the last three inputs (also for T < 3)."""
    r = _rng(9)
    for T in (1, 2, 3, 17):
        C = 12
        x = r.standard_normal((T, C))
        st = r.standard_normal((C, 3))
        w = r.standard_normal((C, 4))
        y, ns = oracle.causal_conv_silu(x, st, w)
        for c in range(C):
            xx = np.concatenate([st[c], x[:, c]])
            pre = np.convolve(xx, w[c, ::-1], mode="valid")
            np.testing.assert_allclose(y[:, c], pre * scipy.special.expit(pre), rtol=1e-13, atol=1e-15)
            np.testing.assert_array_equal(ns[c], xx[-3:])


def test_l2_and_rms_norm_properties():
    """Front end: L2-normalised q/k rows have unit length up to BF16 rounding; the decode
    row (one rounding) and the prefill path (two roundings) differ by at most one BF16
    step. Back end: with w = 1 and a saturated gate the RMS-normalised output has mean
    square 1 up to BF16 rounding, and a zero gate halves it (sigmoid(0) = 1/2)."""
    H, D = 2, 64
    r = _rng(10)
    x = r.standard_normal((5, 3 * H * D))
    st = r.standard_normal((3 * H * D, 3))
    w = r.standard_normal((3 * H * D, 4))
    c, _ = oracle.front_prefill(x, st, w, H, D)
    qn = np.linalg.norm(c[:, :H * D].reshape(5, H, D), axis=-1)
    np.testing.assert_allclose(qn, 1.0, atol=2 ** -7)
    row, _ = oracle.front_decode_row(x[0], st, w, H, D)
    np.testing.assert_allclose(row, c[0], rtol=2 ** -7, atol=1e-30)
    core = r.standard_normal((7, H, D))
    y = oracle.gated_rmsnorm(core, np.full((7, H * D), 60.0), np.ones(D), 1e-6)
    np.testing.assert_allclose(np.mean(y.reshape(7, H, D) ** 2, axis=-1), 1.0, rtol=2 ** -6)
    y0 = oracle.gated_rmsnorm(core, np.zeros((7, H * D)), np.ones(D), 1e-6)
    np.testing.assert_allclose(y0, oracle.bf16_round(y / 2.0), rtol=2 ** -7)


def test_decode_rows_serial_and_snapshots():
    """K rows in one call == K one-row calls on the carried state (bit for bit), and
    snapshot[t] is the state after row t (Glm5NextKdaLayer, decode_k)."""
    from synth import decode_inputs
    H, D, K = 2, 16, 4
    di = decode_inputs(1, H, D, seed=3, K=K)
    args = dict(conv_w=di.conv_w, dt_bias=di.dt_bias, a_log=di.a_log, o_norm_w=di.o_norm, H=H, D=D)
    full = oracle.decode_rows(di.x, di.conv_state[0], g_raw=di.g_raw, b_logit=di.b_logit,
                              out_gate=di.out_gate, h_state=di.s0[0], **args)
    cs, S = di.conv_state[0].double().numpy(), di.s0[0].double().numpy()
    for t in range(K):
        one = oracle.decode_rows(di.x[t:t + 1], cs, g_raw=di.g_raw[t:t + 1], b_logit=di.b_logit[t:t + 1],
                                 out_gate=di.out_gate[t:t + 1], h_state=S, **args)
        assert np.array_equal(one["o_norm_out"][0], full["o_norm_out"][t])
        assert np.array_equal(one["h_state"], full["snapshots"][t][0])
        assert np.array_equal(one["conv_state"], full["snapshots"][t][1])
        cs, S = one["conv_state"], one["h_state"]
    assert np.array_equal(S, full["h_state"]) and np.array_equal(cs, full["conv_state"])


def test_block_prefill_split_equals_whole():
    """Block prefill over T rows == prefill over T1 rows then T2 rows from the carried
    recurrent and conv states (Glm5NextKdaLayer, prefill "from the carried state")."""
    from synth import block_weights, block_hidden
    Wt = block_weights(hidden=64, H=2, D=16, rank=8, seed=5, std=0.2)
    h = block_hidden(23, 64, seed=5)
    hs = np.zeros((2, 16, 16))
    cs = np.zeros((96, 3))
    whole = oracle.block_prefill(Wt, h, hs, cs)
    a = oracle.block_prefill(Wt, h[:10], hs, cs)
    b = oracle.block_prefill(Wt, h[10:], a["h_state"], a["conv_state"])
    np.testing.assert_allclose(np.concatenate([a["final_out"], b["final_out"]]), whole["final_out"],
                               rtol=2 ** -7, atol=1e-6)
    np.testing.assert_allclose(b["h_state"], whole["h_state"], rtol=1e-9, atol=1e-12)
    np.testing.assert_array_equal(b["conv_state"], whole["conv_state"])


def test_block_decode_rows_match_block_prefill():
    """The block decode of K rows (one token at a time: Glm5NextKdaLayer decode / decode_k)
    against the block prefill of the same K tokens: identical projections and conv state; the
    conv output differs only by the prefill's second BF16 rounding of q|k (l2_norm_bf16 in
    place), so the recurrent state and the block output agree to BF16 resolution."""
    from synth import block_weights, block_hidden
    Wt = block_weights(hidden=64, H=2, D=16, rank=8, seed=6, std=0.2)
    h = block_hidden(5, 64, seed=6)
    r = np.random.default_rng(6)
    hs = r.standard_normal((2, 16, 16)) * 0.1
    cs = oracle.bf16_round(r.standard_normal((96, 3)))
    dec = oracle.block_decode(Wt, h, hs, cs)
    pre = oracle.block_prefill(Wt, h, hs, cs)
    for k_ in ("qkv_proj", "g_raw", "b_logit", "out_gate", "conv_state"):
        np.testing.assert_array_equal(dec[k_], pre[k_])
    assert np.all(np.abs(dec["conv_out"] - pre["conv_out"]) <= 2 * 2.0 ** -7 * np.abs(pre["conv_out"]) + 1e-30)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)  # noqa: E731
    assert rel(dec["h_state"], pre["h_state"]) <= 2e-2
    assert rel(dec["final_out"], pre["final_out"]) <= 2e-2
    # decode_k over K rows == K serial one-row decodes (bit for bit), snapshots included
    S, c = hs, cs
    for t in range(5):
        one = oracle.block_decode(Wt, h[t:t + 1], S, c)
        np.testing.assert_array_equal(one["final_out"][0], dec["final_out"][t])
        np.testing.assert_array_equal(one["h_state"], dec["snapshots"][t][0])
        S, c = one["h_state"], one["conv_state"]
