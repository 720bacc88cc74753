"""Pins of the fp64 CPU oracle against facts fixed by the definition and by
mathematics, independent of the oracle's own code.

The step (gated delta rule, the rank-1 update with decay of "GDN tuning limits
on Kunlun XPU", section 二 背景):
    S <- alpha S;  delta = beta (v - S^T k);  S <- S + k delta^T;  o = scale S^T q
Each pin is chosen so that a plausible slip (a dropped decay or beta, a sign
flip in v - S^T k, o read before the update, a transposed S, a wrong GQA map,
a wrong conv tap order, a wrong gate sign) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x)


# ---- the recurrence ---------------------------------------------------------


def test_identity_alpha1_beta0_leaves_state_bit_exact():
    r = _rng(1)
    B, T, H, dk, dv = 2, 3, 2, 16, 8
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    v = r.standard_normal((B, T, H, dv))
    g = np.zeros((B, T, H))
    beta = np.zeros((B, T, H))
    state = r.standard_normal((B, H, dv, dk))
    s0 = state.copy()
    out, rc = oracle.decode_step(q, k, v, g, beta, state, np.arange(B), scale=0.5,
                                 qk_l2norm=False)
    assert rc == 0
    assert np.array_equal(state, s0)
    # o = scale * S^T q, via numpy's matmul on the math-layout S (dk x dv)
    for b in range(B):
        for h in range(H):
            S = s0[b, h].T
            for t in range(T):
                np.testing.assert_allclose(out[b, t, h], 0.5 * (S.T @ q[b, t, h]),
                                           rtol=0, atol=1e-13)


def test_projection_beta1_unit_k_reaches_v():
    """beta = 1 and |k| = 1 make the updated S satisfy S^T k = v exactly; with
    q = k the output is scale * v, which also fails if o were read before the
    update."""
    r = _rng(2)
    dk, dv, H = 32, 16, 3
    k = np.stack([_unit(r.standard_normal(dk)) for _ in range(H)])[None, None]
    v = r.standard_normal((1, 1, H, dv))
    g = r.uniform(-0.5, 0.0, (1, 1, H))
    beta = np.ones((1, 1, H))
    state = r.standard_normal((1, H, dv, dk))
    out, rc = oracle.decode_step(k, k, v, g, beta, state, [0], scale=0.25,
                                 qk_l2norm=False)
    assert rc == 0
    for h in range(H):
        S = state[0, h].T  # math layout dk x dv
        np.testing.assert_allclose(S.T @ k[0, 0, h], v[0, 0, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(out[0, 0, h], 0.25 * v[0, 0, h], rtol=0, atol=1e-12)


def test_decay_only_is_product_of_alphas():
    r = _rng(3)
    B, T, H, dk, dv = 1, 6, 2, 8, 4
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    v = r.standard_normal((B, T, H, dv))
    g = r.uniform(-0.5, 0.0, (B, T, H))
    beta = np.zeros((B, T, H))
    state = r.standard_normal((1, H, dv, dk))
    s0 = state.copy()
    out, _ = oracle.decode_step(q, k, v, g, beta, state, [0], qk_l2norm=True, eps=0.0)
    scale = 1.0 / math.sqrt(dk)
    for h in range(H):
        cum = 1.0
        for t in range(T):
            cum *= math.exp(g[0, t, h])
            qn = _unit(q[0, t, h])
            np.testing.assert_allclose(out[0, t, h], scale * cum * (s0[0, h] @ qn),
                                       rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(state[0, h], cum * s0[0, h], rtol=1e-13, atol=0)


@pytest.mark.parametrize("dk,dv", [(2, 2), (4, 4), (8, 8), (4, 2), (2, 8)])
def test_recurrence_equals_unrolled_product_form(dk, dv):
    """S_t = A_t S_{t-1} + beta_t k_t v_t^T with A_t = alpha_t (I - beta_t k_t k_t^T),
    expanded as S_T = (A_T..A_1) S_0 + sum_t (A_T..A_{t+1}) beta_t k_t v_t^T and
    evaluated with explicit dk x dk matrix products (brute force)."""
    r = _rng(100 + dk * 10 + dv)
    T = 5
    q = r.standard_normal((1, T, 1, dk))
    k = r.standard_normal((1, T, 1, dk))
    v = r.standard_normal((1, T, 1, dv))
    g = r.uniform(-0.5, 0.0, (1, T, 1))
    beta = expit(r.standard_normal((1, T, 1)))
    state = r.standard_normal((1, 1, dv, dk))
    S0 = state[0, 0].T.copy()
    scale = 0.3
    out, _ = oracle.decode_step(q, k, v, g, beta, state, [0], scale=scale,
                                qk_l2norm=True, eps=0.0)
    kn = [_unit(k[0, t, 0]) for t in range(T)]
    qn = [_unit(q[0, t, 0]) for t in range(T)]
    A = [math.exp(g[0, t, 0]) * (np.eye(dk) - beta[0, t, 0] * np.outer(kn[t], kn[t]))
         for t in range(T)]
    for tt in range(1, T + 1):
        P = np.eye(dk)
        for t in range(tt):
            P = A[t] @ P
        St = P @ S0
        for t in range(tt):
            Q = np.eye(dk)
            for s in range(t + 1, tt):
                Q = A[s] @ Q
            St = St + Q @ (beta[0, t, 0] * np.outer(kn[t], v[0, t, 0]))
        np.testing.assert_allclose(out[0, tt - 1, 0], scale * (St.T @ qn[tt - 1]),
                                   rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(state[0, 0].T, St, rtol=1e-11, atol=1e-12)


def test_worked_example_by_hand():
    with open(os.path.join(GOLDEN, "worked_example_dk2_dv2.json")) as f:
        ex = json.load(f)
    dk, dv = ex["dk"], ex["dv"]
    T = len(ex["tokens"])
    q = np.array([tk["q"] for tk in ex["tokens"]]).reshape(1, T, 1, dk)
    k = np.array([tk["k"] for tk in ex["tokens"]]).reshape(1, T, 1, dk)
    v = np.array([tk["v"] for tk in ex["tokens"]]).reshape(1, T, 1, dv)
    g = np.array([tk["g"] for tk in ex["tokens"]]).reshape(1, T, 1)
    beta = np.array([tk["beta"] for tk in ex["tokens"]]).reshape(1, T, 1)
    state = np.ascontiguousarray(np.array(ex["S0_math_dk_by_dv"]).T)[None, None].copy()
    out, rc = oracle.decode_step(q, k, v, g, beta, state, [0], scale=ex["scale"],
                                 qk_l2norm=ex["qk_l2norm"], eps=ex["eps"])
    tol = ex["tolerance_abs"]
    assert rc == 0
    np.testing.assert_allclose(out[0, :, 0], np.array(ex["expected_o"]), atol=tol, rtol=0)
    np.testing.assert_allclose(state[0, 0].T, np.array(ex["expected_S_math_dk_by_dv"]),
                               atol=tol, rtol=0)


def test_in_step_l2norm_matches_prenormalised_inputs():
    r = _rng(4)
    B, T, H, dk, dv = 2, 2, 2, 16, 16
    q = r.standard_normal((B, T, H, dk)) * 3
    k = r.standard_normal((B, T, H, dk)) * 3
    v = r.standard_normal((B, T, H, dv))
    g = r.uniform(-0.5, 0, (B, T, H))
    beta = expit(r.standard_normal((B, T, H)))
    s1 = r.standard_normal((B, H, dv, dk))
    s2 = s1.copy()
    o1, _ = oracle.decode_step(q, k, v, g, beta, s1, np.arange(B), qk_l2norm=True, eps=0.0)
    qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
    kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
    o2, _ = oracle.decode_step(qn, kn, v, g, beta, s2, np.arange(B), qk_l2norm=False)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(s1, s2, rtol=1e-13, atol=1e-15)


def test_default_scale_is_inverse_sqrt_dk():
    r = _rng(5)
    dk, dv = 64, 8
    q = r.standard_normal((1, 1, 1, dk))
    z = np.zeros((1, 1, 1))
    st = r.standard_normal((1, 1, dv, dk))
    o1, _ = oracle.decode_step(q, q, np.zeros((1, 1, 1, dv)), z, z, st.copy(), [0])
    o2, _ = oracle.decode_step(q, q, np.zeros((1, 1, 1, dv)), z, z, st.copy(), [0],
                               scale=0.125)
    np.testing.assert_allclose(o1, o2, rtol=1e-15)


def test_gqa_map_is_contiguous_groups():
    """v-head h reads q/k head h // (H/Hk): equal to a run with q, k repeated
    explicitly per v-head."""
    r = _rng(6)
    B, T, Hk, G, dk, dv = 2, 2, 2, 3, 8, 8
    H = Hk * G
    q = r.standard_normal((B, T, Hk, dk))
    k = r.standard_normal((B, T, Hk, dk))
    v = r.standard_normal((B, T, H, dv))
    g = r.uniform(-0.5, 0, (B, T, H))
    beta = expit(r.standard_normal((B, T, H)))
    s1 = r.standard_normal((B, H, dv, dk))
    s2 = s1.copy()
    o1, _ = oracle.decode_step(q, k, v, g, beta, s1, np.arange(B))
    o2, _ = oracle.decode_step(np.repeat(q, G, axis=2), np.repeat(k, G, axis=2), v, g,
                               beta, s2, np.arange(B))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_slots_padding_and_range():
    r = _rng(7)
    B, T, H, dk, dv, n_slots = 4, 1, 2, 8, 8, 6
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    v = r.standard_normal((B, T, H, dv))
    g = r.uniform(-0.5, 0, (B, T, H))
    beta = expit(r.standard_normal((B, T, H)))
    pool = r.standard_normal((n_slots, H, dv, dk))
    slots = np.array([4, -1, 0, 2], dtype=np.int32)
    st = pool.copy()
    out, rc = oracle.decode_step(q, k, v, g, beta, st, slots)
    assert rc == 0
    assert np.all(out[1] == 0.0)
    for s in (1, 3, 5):  # untouched slots
        assert np.array_equal(st[s], pool[s])
    # a gathered run on a compact pool gives the same numbers
    compact = pool[[4, 0, 2]].copy()
    keep = [0, 2, 3]
    out2, _ = oracle.decode_step(q[keep], k[keep], v[keep], g[keep], beta[keep],
                                 compact, np.arange(3))
    np.testing.assert_array_equal(out2, out[keep])
    np.testing.assert_array_equal(compact, st[[4, 0, 2]])
    # out-of-range slot: reported, row zeroed, pool untouched
    st3 = pool.copy()
    out3, rc3 = oracle.decode_step(q, k, v, g, beta, st3, np.array([0, 6, -2, 1]))
    assert rc3 == oracle.SLOT_RANGE
    assert np.all(out3[1] == 0) and np.all(out3[2] == 0)
    assert np.array_equal(st3[2:], pool[2:])


# ---- scalar and vector pieces of the fused front and epilogue -----------------


def test_scalar_functions_against_library_and_identities():
    xs = np.concatenate([np.linspace(-30, 30, 121), [-700.0, 700.0, 0.0]])
    for x in xs:
        assert oracle.sigmoid(x) == pytest.approx(float(expit(x)), rel=1e-15, abs=1e-300)
        assert oracle.softplus(x) == pytest.approx(float(np.logaddexp(0.0, x)), rel=1e-14,
                                                   abs=1e-300)
        assert oracle.silu(x) == pytest.approx(float(x * expit(x)), rel=1e-15, abs=1e-300)
        # softplus(x) - softplus(-x) = x
        assert oracle.softplus(x) - oracle.softplus(-x) == pytest.approx(x, abs=1e-12)
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-16)
    assert oracle.sigmoid(0.0) == 0.5 and oracle.silu(0.0) == 0.0


def test_gate_closed_forms():
    # A_log = 0 and a + dt_bias = 0: g = -softplus(0) = -ln 2, alpha = 1/2
    assert oracle.gate_g(0.7, 0.0, -0.7) == pytest.approx(-math.log(2.0), rel=1e-15)
    assert math.exp(oracle.gate_g(0.0, 0.0, 0.0)) == pytest.approx(0.5, rel=1e-15)
    # g scales with exp(A_log) and is always <= 0 (alpha in (0, 1])
    assert oracle.gate_g(1.3, math.log(4.0), 0.2) == pytest.approx(
        -4.0 * float(np.logaddexp(0.0, 1.5)), rel=1e-14)
    for a in np.linspace(-10, 10, 41):
        assert oracle.gate_g(a, 0.3, -0.1) < 0.0


def test_conv4_taps_and_dot_product():
    r = _rng(8)
    cs = r.standard_normal(3)
    x = float(r.standard_normal())
    for m in range(4):
        w = np.zeros(4)
        w[m] = 1.0
        want = cs[m] if m < 3 else x
        assert oracle.conv4(cs, x, w) == want
    for _ in range(10):
        w = r.standard_normal(4)
        assert oracle.conv4(cs, x, w) == pytest.approx(
            float(np.dot(w, np.append(cs, x))), rel=1e-14, abs=1e-15)


def test_l2norm_and_gated_rmsnorm_special_cases():
    x = np.array([3.0, 4.0])
    np.testing.assert_allclose(oracle.l2norm(x), [0.6, 0.8], rtol=1e-15)
    r = _rng(9)
    dv = 16
    z = r.standard_normal(dv)
    w = np.ones(dv)
    for c in (2.5, -0.01):
        y = oracle.gated_rmsnorm(np.full(dv, c), z, w, eps=0.0)
        np.testing.assert_allclose(y, math.copysign(1.0, c) * z * expit(z), rtol=1e-14)
    # scale invariance of the norm part, linearity in w
    o = r.standard_normal(dv)
    w2 = r.standard_normal(dv)
    np.testing.assert_allclose(oracle.gated_rmsnorm(7.0 * o, z, w2, eps=0.0),
                               oracle.gated_rmsnorm(o, z, w2, eps=0.0), rtol=1e-13)
    rms = math.sqrt(np.mean(o * o))
    np.testing.assert_allclose(oracle.gated_rmsnorm(o, z, w2, eps=0.0),
                               o / rms * w2 * z * expit(z), rtol=1e-13)


def _fused_inputs(r, B, Hk, H, dk, dv, n_slots):
    C = 2 * Hk * dk + H * dv
    return dict(
        mixed_x=r.standard_normal((B, C)),
        conv_state=r.standard_normal((n_slots, C, 3)),
        conv_w=r.standard_normal((C, 4)) * 0.5,
        a=r.standard_normal((B, H)),
        b=r.standard_normal((B, H)),
        A_log=np.log(r.uniform(1, 16, H)),
        dt_bias=r.standard_normal(H) * 0.5,
        z=r.standard_normal((B, H * dv)),
        norm_w=1.0 + 0.1 * r.standard_normal(dv),
        state=r.standard_normal((n_slots, H, dv, dk)) * 0.02,
    )


def test_fused_reduces_to_plain_step_with_identity_conv():
    """conv weight e_3 makes the conv the identity on x; A_log = 0 with
    a = -dt_bias gives alpha = 1/2 and b = 0 gives beta = 1/2.  The fused step
    must then equal the plain step fed with silu(x) split as [q | k | v], with
    q/k repeated per v-head, followed by the gated RMSNorm."""
    r = _rng(10)
    B, Hk, G, dk, dv, n_slots = 3, 2, 3, 8, 4, 4
    H = Hk * G
    inp = _fused_inputs(r, B, Hk, H, dk, dv, n_slots)
    C = inp["mixed_x"].shape[1]
    inp["conv_w"] = np.tile(np.array([0.0, 0.0, 0.0, 1.0]), (C, 1))
    inp["A_log"] = np.zeros(H)
    inp["a"] = np.tile(-inp["dt_bias"], (B, 1))
    inp["b"] = np.zeros((B, H))
    slots = np.array([2, 0, 3], dtype=np.int32)
    st_f = inp["state"].copy()
    cs_f = inp["conv_state"].copy()
    out_f, rc = oracle.fused_step(inp["mixed_x"], cs_f, inp["conv_w"], inp["a"], inp["b"],
                                  inp["A_log"], inp["dt_bias"], inp["z"], inp["norm_w"],
                                  st_f, slots, Hk=Hk, H=H, dk=dk, dv=dv, norm_eps=0.0)
    assert rc == 0
    xs = inp["mixed_x"] * expit(inp["mixed_x"])
    q = xs[:, : Hk * dk].reshape(B, 1, Hk, dk)
    k = xs[:, Hk * dk: 2 * Hk * dk].reshape(B, 1, Hk, dk)
    v = xs[:, 2 * Hk * dk:].reshape(B, 1, H, dv)
    st_p = inp["state"].copy()
    o, _ = oracle.decode_step(np.repeat(q, G, axis=2), np.repeat(k, G, axis=2), v,
                              np.full((B, 1, H), -math.log(2.0)), np.full((B, 1, H), 0.5),
                              st_p, slots)
    np.testing.assert_allclose(st_f, st_p, rtol=1e-13, atol=1e-15)
    for b in range(B):
        for h in range(H):
            want = oracle.gated_rmsnorm(o[b, 0, h], inp["z"][b, h * dv:(h + 1) * dv],
                                        inp["norm_w"], eps=0.0)
            np.testing.assert_allclose(out_f[b, h], want, rtol=1e-12, atol=1e-14)
    # conv state shifted: [cs1, cs2, x], oldest first
    for b, s in enumerate(slots):
        np.testing.assert_array_equal(cs_f[s, :, 0], inp["conv_state"][s, :, 1])
        np.testing.assert_array_equal(cs_f[s, :, 1], inp["conv_state"][s, :, 2])
        np.testing.assert_array_equal(cs_f[s, :, 2], inp["mixed_x"][b])
    untouched = [s for s in range(n_slots) if s not in slots]
    for s in untouched:
        np.testing.assert_array_equal(cs_f[s], inp["conv_state"][s])
        np.testing.assert_array_equal(st_f[s], inp["state"][s])


def test_fused_conv_uses_previous_inputs_oldest_first():
    """Three fused calls with conv weight e_0 on a zero-initialised conv state:
    the call n conv output is the input of call n-3 (zero before that)."""
    r = _rng(11)
    B, Hk, H, dk, dv = 1, 1, 1, 4, 4
    inp = _fused_inputs(r, B, Hk, H, dk, dv, 1)
    C = inp["mixed_x"].shape[1]
    cs = np.zeros((1, C, 3))
    w = np.tile(np.array([1.0, 0.0, 0.0, 0.0]), (C, 1))
    xs = [r.standard_normal((B, C)) for _ in range(4)]
    st = inp["state"].copy()
    outs = []
    for n in range(4):
        if n == 3:
            st_before = st.copy()
        o, _ = oracle.fused_step(xs[n], cs, w, inp["a"], inp["b"], inp["A_log"],
                                 inp["dt_bias"], inp["z"], inp["norm_w"], st, [0],
                                 Hk=Hk, H=H, dk=dk, dv=dv)
        outs.append(o)
    # call 3 sees xs[0] through tap 0: same as an identity conv (tap 3) fed xs[0]
    w3 = np.tile(np.array([0.0, 0.0, 0.0, 1.0]), (C, 1))
    o3, _ = oracle.fused_step(xs[0], np.zeros((1, C, 3)), w3, inp["a"], inp["b"],
                              inp["A_log"], inp["dt_bias"], inp["z"], inp["norm_w"],
                              st_before, [0], Hk=Hk, H=H, dk=dk, dv=dv)
    np.testing.assert_array_equal(o3, outs[3])
    # calls 0..2 see an all-zero conv output -> v = 0, q = k = 0 -> o = alpha S^T 0 = 0
    for n in range(3):
        assert np.all(outs[n] == 0.0)
    np.testing.assert_array_equal(cs[0, :, 0], xs[1][0])
    np.testing.assert_array_equal(cs[0, :, 2], xs[3][0])


def test_fused_padding_rows():
    r = _rng(12)
    B, Hk, H, dk, dv, n_slots = 3, 1, 2, 4, 4, 3
    inp = _fused_inputs(r, B, Hk, H, dk, dv, n_slots)
    st = inp["state"].copy()
    cs = inp["conv_state"].copy()
    out, rc = oracle.fused_step(inp["mixed_x"], cs, inp["conv_w"], inp["a"], inp["b"],
                                inp["A_log"], inp["dt_bias"], inp["z"], inp["norm_w"], st,
                                [-1, 1, -1], Hk=Hk, H=H, dk=dk, dv=dv)
    assert rc == 0
    assert np.all(out[0] == 0) and np.all(out[2] == 0) and np.any(out[1] != 0)
    for s in (0, 2):
        np.testing.assert_array_equal(st[s], inp["state"][s])
        np.testing.assert_array_equal(cs[s], inp["conv_state"][s])


# ---- storage rounding of the state pool ---------------------------------------


def test_fp16_rounding_matches_numpy_including_ties_and_subnormals():
    r = _rng(20)
    xs = np.concatenate([
        r.standard_normal(2000) * 10.0 ** r.uniform(-9, 5, 2000),
        [1 + 2 ** -11, 1 + 3 * 2 ** -11, 2 ** -24, 3 * 2 ** -25, 2 ** -25, 65504.0, 65519.99,
         65520.0, -65520.0, 6.1e-5, -0.0, 0.0],
    ])
    for x in xs:
        want = float(np.float16(x))
        got = oracle.round_storage(x, "fp16")
        assert got == want or (math.isnan(want) and math.isnan(got)), (x, got, want)


def test_fp32_rounding_matches_numpy():
    r = _rng(21)
    xs = r.standard_normal(2000) * 10.0 ** r.uniform(-40, 38, 2000)
    for x in xs:
        assert oracle.round_storage(x, "fp32") == float(np.float32(x)), x


def test_bf16_rounding_matches_torch_on_fp32_values():
    import torch
    r = _rng(22)
    xs = (r.standard_normal(4000) * 10.0 ** r.uniform(-38, 38, 4000)).astype(np.float32)
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -20],
                    dtype=np.float32)
    xs = np.concatenate([xs, ties])
    want = torch.from_numpy(xs).to(torch.bfloat16).to(torch.float64).numpy()
    for x, w in zip(xs, want):
        assert oracle.round_storage(float(x), "bf16") == float(w), (x, w)
    # ties to even by hand: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7
    assert oracle.round_storage(1 + 2 ** -8, "bf16") == 1.0
    assert oracle.round_storage(1 + 3 * 2 ** -8, "bf16") == 1 + 2 ** -6


def test_decode_step_rounds_the_state_once_per_call():
    r = _rng(23)
    B, T, H, dk, dv = 1, 3, 2, 8, 4
    args = [r.standard_normal((B, T, H, dk)), r.standard_normal((B, T, H, dk)),
            r.standard_normal((B, T, H, dv)), r.uniform(-0.5, 0, (B, T, H)),
            expit(r.standard_normal((B, T, H)))]
    s0 = r.standard_normal((1, H, dv, dk))
    s_exact, s_round = s0.copy(), s0.copy()
    o1, _ = oracle.decode_step(*args, s_exact, [0])
    o2, _ = oracle.decode_step(*args, s_round, [0], state_round="bf16")
    np.testing.assert_array_equal(o1, o2)  # outputs use the unrounded in-call state
    want = np.vectorize(lambda x: oracle.round_storage(x, "bf16"))(s_exact)
    np.testing.assert_array_equal(s_round, want)


# ---- speculative-decoding state handling ----------------------------------------


def _spec_inputs(seed, B=3, T=4, H=2, dk=8, dv=4):
    r = _rng(seed)
    return dict(q=r.standard_normal((B, T, H, dk)), k=r.standard_normal((B, T, H, dk)),
                v=r.standard_normal((B, T, H, dv)), g=r.uniform(-0.5, 0, (B, T, H)),
                beta=expit(r.standard_normal((B, T, H)))), r


def _prefix(a, n, b):
    return {key: val[b:b + 1, :n] for key, val in a.items()}


def test_accept_length_commit_equals_a_call_on_the_accepted_prefix():
    a, r = _spec_inputs(30)
    B, T, H, dv, dk = 3, 4, 2, 4, 8
    pool = r.standard_normal((5, H, dv, dk))
    slots = np.array([4, 0, 2], dtype=np.int32)
    n_acc = np.array([2, 0, 4], dtype=np.int32)
    st = pool.copy()
    out, rc = oracle.decode_step_spec(*a.values(), st, slots, n_accept=n_acc)
    assert rc == 0
    full, _ = oracle.decode_step(*a.values(), pool.copy(), slots)
    np.testing.assert_array_equal(out, full)  # outputs of every token, as without commit
    for b in range(B):
        want = pool[slots[b]].copy()[None]
        if n_acc[b] > 0:
            oracle.decode_step(*_prefix(a, n_acc[b], b).values(), want, [0])
        np.testing.assert_array_equal(st[slots[b]], want[0])
    np.testing.assert_array_equal(st[[1, 3]], pool[[1, 3]])


def test_token_snapshots_hold_every_prefix_state():
    a, r = _spec_inputs(31)
    B, T, H, dv, dk = 3, 4, 2, 4, 8
    pool = r.standard_normal((3 + B * T, H, dv, dk))
    slots = np.array([0, 1, 2], dtype=np.int32)
    tsl = (3 + np.arange(B * T, dtype=np.int32)).reshape(B, T)
    tsl[1, 2] = -1
    st = pool.copy()
    out, rc = oracle.decode_step_spec(*a.values(), st, slots, token_slots=tsl)
    assert rc == 0
    np.testing.assert_array_equal(st[:3], pool[:3])  # the source slots are not written
    for b in range(B):
        for t in range(T):
            want = pool[slots[b]].copy()[None]
            oracle.decode_step(*_prefix(a, t + 1, b).values(), want, [0])
            if tsl[b, t] >= 0:
                np.testing.assert_array_equal(st[tsl[b, t]], want[0])
    np.testing.assert_array_equal(st[tsl[1, 2] if tsl[1, 2] >= 0 else 3 + 6], pool[3 + 6])


def test_spec_modes_report_bad_values():
    a, r = _spec_inputs(32)
    pool = r.standard_normal((4, 2, 4, 8))
    st = pool.copy()
    _, rc = oracle.decode_step_spec(*a.values(), st, [0, 1, 2], n_accept=[5, -1, 1])
    assert rc & oracle.ACCEPT_RANGE
    np.testing.assert_array_equal(st[[0, 1]], pool[[0, 1]])
    assert not np.array_equal(st[2], pool[2])
    tsl = np.full((3, 4), -1, dtype=np.int32)
    tsl[0, 0] = 9
    _, rc = oracle.decode_step_spec(*a.values(), pool.copy(), [0, 1, 2], token_slots=tsl)
    assert rc & oracle.SLOT_RANGE


# ---- prefill over packed variable-length sequences ------------------------------


def _prefill_inputs(seed, lens, H=2, Hk=2, dk=8, dv=4, n_slots=None):
    r = _rng(seed)
    total = int(sum(lens))
    d = dict(q=r.standard_normal((total, Hk, dk)), k=r.standard_normal((total, Hk, dk)),
             v=r.standard_normal((total, H, dv)), g=r.uniform(-0.5, 0, (total, H)),
             beta=expit(r.standard_normal((total, H))))
    pool = r.standard_normal((n_slots or len(lens), H, dv, dk))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return d, pool, cu


def test_prefill_equals_one_multi_token_decode_call_per_sequence():
    lens = [5, 1, 9, 3]
    d, pool, cu = _prefill_inputs(40, lens, n_slots=6)
    slots = np.array([3, 0, 5, 1], dtype=np.int32)
    st = pool.copy()
    out, rc = oracle.prefill(*d.values(), st, slots, cu)
    assert rc == 0
    for n, L in enumerate(lens):
        t0, t1 = cu[n], cu[n + 1]
        ref = pool[slots[n]].copy()[None]
        o, _ = oracle.decode_step(d["q"][None, t0:t1], d["k"][None, t0:t1], d["v"][None, t0:t1],
                                  d["g"][None, t0:t1], d["beta"][None, t0:t1], ref, [0])
        np.testing.assert_array_equal(out[t0:t1], o[0])
        np.testing.assert_array_equal(st[slots[n]], ref[0])
    np.testing.assert_array_equal(st[[2, 4]], pool[[2, 4]])


def test_prefill_from_zero_state_and_padding():
    d, pool, cu = _prefill_inputs(41, [4, 6])
    st = pool.copy()
    out, _ = oracle.prefill(*d.values(), st, [0, -1], cu, initial_state=False)
    ref = np.zeros_like(pool[:1])
    o, _ = oracle.decode_step(d["q"][None, :4], d["k"][None, :4], d["v"][None, :4],
                              d["g"][None, :4], d["beta"][None, :4], ref, [0])
    np.testing.assert_array_equal(out[:4], o[0])
    np.testing.assert_array_equal(st[0], ref[0])
    assert np.all(out[4:] == 0) and np.array_equal(st[1], pool[1])


@pytest.mark.parametrize("L,C", [(7, 4), (12, 4), (5, 8), (16, 16)])
def test_chunkwise_form_of_the_recurrence(L, C):
    """The chunked prefill computes, per chunk of C tokens starting from S0:
         gamma_i = exp(sum_{t0<=j<=i} g_j)  (cumulative decay in the chunk)
         A_ij = beta_i (k_i.k_j) gamma_i/gamma_j   for j < i
         Delta = (I + A)^-1 diag(beta) (V - diag(gamma) K S0)
         O = scale (diag(gamma) Q S0 + P Delta),  P_ij = (q_i.k_j) gamma_i/gamma_j, j <= i
         S_end = gamma_C S0 + (K * gamma_C/gamma)^T Delta
       (S is dk x dv, rows of K, Q are normalised tokens).  Evaluated here with
       numpy's dense solve, it must equal the oracle's token-by-token recurrence."""
    d, pool, cu = _prefill_inputs(42 + L + C, [L], H=1, Hk=1, dk=8, dv=4)
    st = pool.copy()
    out, _ = oracle.prefill(*d.values(), st, [0], cu, scale=0.5, eps=0.0)
    K = d["k"][:, 0] / np.linalg.norm(d["k"][:, 0], axis=1, keepdims=True)
    Q = d["q"][:, 0] / np.linalg.norm(d["q"][:, 0], axis=1, keepdims=True)
    V, g, beta = d["v"][:, 0], d["g"][:, 0], d["beta"][:, 0]
    S = pool[0, 0].T.copy()  # math layout dk x dv
    O = np.zeros((L, V.shape[1]))
    for c0 in range(0, L, C):
        sl = slice(c0, min(c0 + C, L))
        Kc, Qc, Vc, bc = K[sl], Q[sl], V[sl], beta[sl]
        G = np.cumsum(g[sl])
        ratio = np.exp(G[:, None] - G[None, :])
        n = Kc.shape[0]
        A = np.tril(bc[:, None] * (Kc @ Kc.T) * ratio, -1)
        Delta = np.linalg.solve(np.eye(n) + A, bc[:, None] * (Vc - np.exp(G)[:, None] * (Kc @ S)))
        P = np.tril((Qc @ Kc.T) * ratio)
        O[sl] = 0.5 * (np.exp(G)[:, None] * (Qc @ S) + P @ Delta)
        S = np.exp(G[-1]) * S + (Kc * np.exp(G[-1] - G)[:, None]).T @ Delta
    np.testing.assert_allclose(out[:, 0], O, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(st[0, 0].T, S, rtol=1e-10, atol=1e-12)


# ---- low-rank sliding-window decode ----------------------------------------------


def _lr_window(n_slots, H, R, dk, dv):
    return (np.zeros((n_slots, H, R, dk)), np.zeros((n_slots, H, R, dv)),
            np.zeros((n_slots, H, R)), np.zeros((n_slots, H), dtype=np.int32))


def _lr_tokens(r, B, T, H, dk, dv):
    return (r.standard_normal((B, T, H, dk)), r.standard_normal((B, T, H, dk)),
            r.standard_normal((B, T, H, dv)), r.uniform(-0.5, 0, (B, T, H)),
            expit(r.standard_normal((B, T, H))))


def test_lowrank_equals_full_rank_until_the_window_wraps():
    """From an empty window and a zero full-rank state, while no update has
    been evicted the window holds every update ever made, so the two
    recurrences are the same map."""
    r = _rng(50)
    B, H, R, dk, dv = 2, 3, 8, 8, 4
    win = _lr_window(B, H, R, dk, dv)
    full = np.zeros((B, H, dv, dk))
    for step in range(R):
        toks = _lr_tokens(r, B, 1, H, dk, dv)
        o_lr, _ = oracle.lowrank_decode_step(*toks, *win, np.arange(B))
        o_full, _ = oracle.decode_step(*toks, full, np.arange(B))
        np.testing.assert_allclose(o_lr, o_full, rtol=1e-12, atol=1e-14)
    # T > 1 in one call crosses no eviction either
    win2 = _lr_window(B, H, R, dk, dv)
    full2 = np.zeros((B, H, dv, dk))
    toks = _lr_tokens(r, B, R, H, dk, dv)
    o_lr, _ = oracle.lowrank_decode_step(*toks, *win2, np.arange(B))
    o_full, _ = oracle.decode_step(*toks, full2, np.arange(B))
    np.testing.assert_allclose(o_lr, o_full, rtol=1e-12, atol=1e-14)
    assert np.all(win2[3] == R)


def test_lowrank_window_matches_brute_force_after_wrapping():
    """After the window wraps, rebuild S = sum_j c_j k_j u_j^T from an
    explicit list of the last R updates (with their accumulated decay) and
    apply the definition's step to it."""
    r = _rng(51)
    H, R, dk, dv = 2, 4, 6, 5
    win = _lr_window(1, H, R, dk, dv)
    hist = [[] for _ in range(H)]  # per head: list of [c, k, u]
    for step in range(3 * R + 1):
        q, k, v, g, beta = _lr_tokens(r, 1, 1, H, dk, dv)
        o, _ = oracle.lowrank_decode_step(q, k, v, g, beta, *win, [0], qk_l2norm=True, eps=0.0)
        for h in range(H):
            kn = k[0, 0, h] / np.linalg.norm(k[0, 0, h])
            qn = q[0, 0, h] / np.linalg.norm(q[0, 0, h])
            a = np.exp(g[0, 0, h])
            for e in hist[h]:
                e[0] *= a
            S = sum((e[0] * np.outer(e[1], e[2]) for e in hist[h]), np.zeros((dk, dv)))
            delta = beta[0, 0, h] * (v[0, 0, h] - S.T @ kn)
            hist[h].append([1.0, kn, delta])
            if len(hist[h]) > R:
                hist[h].pop(0)
            S = sum((e[0] * np.outer(e[1], e[2]) for e in hist[h]), np.zeros((dk, dv)))
            np.testing.assert_allclose(o[0, 0, h], (S.T @ qn) / np.sqrt(dk), rtol=1e-12,
                                       atol=1e-14)
    assert np.all(win[3] == 3 * R + 1)


def test_lowrank_window_of_one_is_the_last_update():
    """R = 1: the window holds only the newest update, so after a step the
    state is k delta^T and o = scale (k.q) delta, with
    delta = beta (v - alpha (k_prev.k) delta_prev)."""
    r = _rng(52)
    dk, dv = 4, 3
    win = _lr_window(1, 1, 1, dk, dv)
    prev_k, prev_d = None, None
    for step in range(5):
        q, k, v, g, beta = _lr_tokens(r, 1, 1, 1, dk, dv)
        o, _ = oracle.lowrank_decode_step(q, k, v, g, beta, *win, [0], eps=0.0)
        kn = k[0, 0, 0] / np.linalg.norm(k[0, 0, 0])
        qn = q[0, 0, 0] / np.linalg.norm(q[0, 0, 0])
        p = 0.0 if prev_k is None else np.exp(g[0, 0, 0]) * (prev_k @ kn) * prev_d
        delta = beta[0, 0, 0] * (v[0, 0, 0] - p)
        np.testing.assert_allclose(o[0, 0, 0], (kn @ qn) * delta / np.sqrt(dk), rtol=1e-12,
                                   atol=1e-14)
        prev_k, prev_d = kn, delta


# ---- low-rank window over whole prompts --------------------------------------------


def _lr_prefill_inputs(seed, lens, H=2, dk=8, dv=4):
    r = _rng(seed)
    total = int(sum(lens))
    d = dict(q=r.standard_normal((total, H, dk)), k=r.standard_normal((total, H, dk)),
             v=r.standard_normal((total, H, dv)), g=r.uniform(-0.5, 0, (total, H)),
             beta=expit(r.standard_normal((total, H))))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return d, cu


def _lr_full_window(r, n_slots, H, R, dk, dv, count):
    k = r.standard_normal((n_slots, H, R, dk))
    return [k / np.linalg.norm(k, axis=-1, keepdims=True), 0.1 * r.standard_normal((n_slots, H, R, dv)),
            r.uniform(0.05, 1.0, (n_slots, H, R)), np.full((n_slots, H), count, dtype=np.int32)]


def test_lowrank_prefill_equals_one_token_decode_calls():
    """The low-rank prefill of a prompt is the low-rank decode step applied
    to its tokens one call at a time (bit for bit: the same arithmetic)."""
    r = _rng(60)
    lens, H, R, dk, dv = [5, 19, 1, 11], 2, 8, 8, 4
    d, cu = _lr_prefill_inputs(61, lens, H, dk, dv)
    win0 = _lr_full_window(r, 5, H, R, dk, dv, count=3 * R + 2)
    win0[3][2] = 3  # one slot whose window is not full yet
    slots = np.array([4, 2, -1, 0], dtype=np.int32)
    win = [w.copy() for w in win0]
    out, rc = oracle.lowrank_prefill(*d.values(), *win, slots, cu)
    assert rc == 0
    ref = [w.copy() for w in win0]
    for n in range(len(lens)):
        t0, t1 = cu[n], cu[n + 1]
        if slots[n] < 0:
            assert np.all(out[t0:t1] == 0)
            continue
        for t in range(t0, t1):
            toks = [d[x][None, t:t + 1] for x in ("q", "k", "v", "g", "beta")]
            o, _ = oracle.lowrank_decode_step(*toks, *ref, [slots[n]])
            np.testing.assert_array_equal(out[t], o[0, 0])
    for a, b in zip(win, ref):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(win[0][[1, 3]], win0[0][[1, 3]])  # untouched slots


def _lr_chunk_form(K, Q, V, g, beta, Kw, Uw, cw, n0, R, C, scale):
    """The low-rank window over one prompt in chunks of C tokens (C >= R).
    The window entering a chunk that starts at token a holds the last
    min(R, n0 + a) updates, each with its weight w at the chunk start; token
    t = a + tau of the chunk sees entering entry e (the e-th oldest of R)
    when e >= tau (the R most recent updates before t), and the chunk's own
    tokens s with t - R <= s < t.  With Gamma the decay from the chunk start:
      (I + A) Delta = diag(beta) (V - M),
        A_ts = beta_t exp(Gamma_t - Gamma_s) (k_s . k_t)  (s < t, t - s <= R)
        M_t  = sum_{e >= tau} w_e exp(Gamma_t) (k_e . k_t) u_e
      O_t = scale (sum_{e > tau} w_e exp(Gamma_t) (k_e . q_t) u_e
                   + sum_{s <= t, t - s < R} exp(Gamma_t - Gamma_s) (k_s . q_t) Delta_s)
    and the window leaving it is the last R of [entering entries, the chunk's
    tokens] with their weights at the chunk end.  Entries are kept oldest
    first; missing ones (a window not yet full) weigh 0."""
    L, dk = K.shape
    dv = V.shape[1]
    # entering entries, oldest first, padded to R with zero weight
    ek = np.zeros((R, dk)); eu = np.zeros((R, dv)); ew = np.zeros(R)
    m = min(n0, R)
    ek[R - m:], eu[R - m:], ew[R - m:] = Kw[-m:] if m else ek[:0], Uw[-m:] if m else eu[:0], \
        cw[-m:] if m else ew[:0]
    O = np.zeros((L, dv))
    for a in range(0, L, C):
        n = min(C, L - a)
        Kc, Qc, Vc, bc = K[a:a + n], Q[a:a + n], V[a:a + n], beta[a:a + n]
        Gm = np.cumsum(g[a:a + n])
        tau = np.arange(n)
        vis_e = np.arange(R)[None, :] >= tau[:, None]            # entering entry e seen by t
        vis_o = np.arange(R)[None, :] > tau[:, None]
        dist = tau[:, None] - tau[None, :]
        band = (dist > 0) & (dist <= R)
        band_o = (dist >= 0) & (dist < R)
        ratio = np.exp(Gm[:, None] - Gm[None, :])
        M = (vis_e * np.exp(Gm)[:, None] * (Kc @ ek.T) * ew[None, :]) @ eu
        A = bc[:, None] * ratio * (Kc @ Kc.T) * band
        Delta = np.linalg.solve(np.eye(n) + A, bc[:, None] * (Vc - M))
        O[a:a + n] = scale * ((vis_o * np.exp(Gm)[:, None] * (Qc @ ek.T) * ew[None, :]) @ eu
                              + (ratio * (Qc @ Kc.T) * band_o) @ Delta)
        # the window leaving the chunk
        allk = np.concatenate([ek, Kc]); allu = np.concatenate([eu, Delta])
        allw = np.concatenate([ew * np.exp(Gm[-1]), np.exp(Gm[-1] - Gm)])
        ek, eu, ew = allk[-R:], allu[-R:], allw[-R:]
    return O, ek, eu, ew


@pytest.mark.parametrize("L,C,R,n0", [(20, 8, 8, 0), (20, 8, 4, 0), (13, 8, 8, 30),
                                      (13, 8, 8, 3), (9, 4, 4, 2), (16, 16, 8, 12)])
def test_lowrank_prefill_chunk_form(L, C, R, n0):
    """The chunked form of the low-rank window above, evaluated with numpy's
    dense solve, equals the oracle's token-by-token window (outputs and the
    window left behind, read in update order)."""
    r = _rng(70 + L + C + R + n0)
    dk, dv = 8, 4
    d, cu = _lr_prefill_inputs(71 + L, [L], 1, dk, dv)
    win = _lr_full_window(r, 1, 1, R, dk, dv, count=n0)
    # entries of the initial window in update order, oldest first
    m = min(n0, R)
    order = [(n0 - m + i) % R for i in range(m)]
    Kw, Uw, cw = (win[0][0, 0][order], win[1][0, 0][order], win[2][0, 0][order])
    K = d["k"][:, 0] / np.linalg.norm(d["k"][:, 0], axis=1, keepdims=True)
    Q = d["q"][:, 0] / np.linalg.norm(d["q"][:, 0], axis=1, keepdims=True)
    O, ek, eu, ew = _lr_chunk_form(K, Q, d["v"][:, 0], d["g"][:, 0], d["beta"][:, 0], Kw, Uw, cw,
                                   n0, R, C, 0.5)
    out, _ = oracle.lowrank_prefill(*d.values(), *win, [0], cu, scale=0.5, eps=0.0)
    np.testing.assert_allclose(out[:, 0], O, rtol=1e-10, atol=1e-12)
    cnt = n0 + L
    m2 = min(cnt, R)
    order2 = [(cnt - m2 + i) % R for i in range(m2)]
    np.testing.assert_allclose(win[0][0, 0][order2], ek[R - m2:], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(win[1][0, 0][order2], eu[R - m2:], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(win[2][0, 0][order2], ew[R - m2:], rtol=1e-10, atol=1e-14)
    assert win[3][0, 0] == cnt


def test_lowrank_prefill_from_an_empty_window_equals_the_full_rank_prefill():
    """Started empty, a prompt no longer than R evicts nothing: the low-rank
    prefill is then the full-rank prefill from a zero state."""
    lens, H, R, dk, dv = [6, 8], 2, 8, 8, 4
    d, cu = _lr_prefill_inputs(80, lens, H, dk, dv)
    win = list(_lr_window(2, H, R, dk, dv))
    win[3][:] = 99  # ignored: initial_window=False starts from count 0
    o_lr, _ = oracle.lowrank_prefill(*d.values(), *win, [1, 0], cu, initial_window=False)
    st = np.zeros((2, H, dv, dk))
    o_full, _ = oracle.prefill(*d.values(), st, [1, 0], cu, initial_state=False)
    np.testing.assert_allclose(o_lr, o_full, rtol=1e-12, atol=1e-14)
    assert np.all(win[3][1] == 6) and np.all(win[3][0] == 8)
