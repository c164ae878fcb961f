"""Pins for the fp64 oracle: each test checks it against something other than
itself — a closed form, a special case that reduces to a textbook operation, a
brute-force product of transition matrices, an invariant, or a hand-derived
fixture under ``tests/golden``.  A plausible slip in the oracle (a dropped term,
a wrong sign, reading y before the update, decaying the rank-one term, a
transposed state) fails at least one of them; see the comment on each test.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_inputs(rng, B, T, H, D, s0=True):
    r, k, v = (rng.standard_normal((B, T, H, D)) for _ in range(3))
    x = rng.standard_normal((B, T, H, D))
    kappa = x / np.linalg.norm(x, axis=-1, keepdims=True)
    a_lr = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, D))))
    z = rng.standard_normal((B, T, H, D))
    w_log = -np.log1p(np.exp(-z)) - 0.5
    a, b = -kappa, kappa * a_lr
    S0 = rng.standard_normal((B, H, D, D)) * 0.3 if s0 else None
    return r, w_log, k, v, a, b, S0


def test_linear_attention_closed_form(oracle_mod):
    """a = b = 0 and w = 1 (l = -inf): y_t = S0 r_t + sum_{i<=t} (k_i . r_t) v_i,
    i.e. Y = R S0^T + tril(R K^T) V, the "Q (K^T V)" linear attention of the
    RWKV-7 analysis page.  Catches a transposed state (S0 is not symmetric), a
    read-out before the update (the diagonal of tril would be missing) and a
    wrong v/k role."""
    rng = np.random.default_rng(1)
    B, T, H, D = 2, 23, 3, 64
    r, _, k, v, _, _, S0 = _rand_inputs(rng, B, T, H, D)
    zeros = np.zeros_like(r)
    w_log = np.full_like(r, -np.inf)
    y, sT = oracle_mod.forward(r, w_log, k, v, zeros, zeros, S0)
    for n in range(B):
        for h in range(H):
            R, K, V = r[n, :, h], k[n, :, h], v[n, :, h]
            Y = R @ S0[n, h].T + np.tril(R @ K.T) @ V
            np.testing.assert_allclose(y[n, :, h], Y, rtol=0, atol=1e-10)
            np.testing.assert_allclose(sT[n, h], S0[n, h] + V.T @ K, rtol=0, atol=1e-10)


def test_diagonal_decay_closed_form(oracle_mod):
    """a = b = 0 (diagonal decay only, the RWKV-6 form):
    y_t = sum_{i<=t} v_i ((k_i * prod_{s=i+1..t} w_s) . r_t) + S0 (prod_{s<=t} w_s * r_t).
    Pins the decay index (the token written at t is not decayed at t) and the
    decay formula w = exp(-exp(l))."""
    rng = np.random.default_rng(2)
    B, T, H, D = 1, 12, 2, 16
    r, w_log, k, v, _, _, S0 = _rand_inputs(rng, B, T, H, D)
    zeros = np.zeros_like(r)
    y, sT = oracle_mod.forward(r, w_log, k, v, zeros, zeros, S0)
    w = np.exp(-np.exp(w_log))
    for h in range(H):
        for t in range(T):
            expect = S0[0, h] @ (np.prod(w[0, : t + 1, h], axis=0) * r[0, t, h])
            for i in range(t + 1):
                decay = np.prod(w[0, i + 1: t + 1, h], axis=0) if i < t else np.ones(D)
                expect = expect + v[0, i, h] * np.dot(k[0, i, h] * decay, r[0, t, h])
            np.testing.assert_allclose(y[0, t, h], expect, rtol=0, atol=1e-11)


def test_delta_rule_exact_retrieval(oracle_mod):
    """w = 1, a = -kappa, b = kappa (a_lr = 1), k = kappa unit: the delta rule
    replaces the value stored under kappa, so S_t kappa_t = v_t exactly and with
    r_t = kappa_t the output is v_t (the DeltaNet special case on the RWKV-7
    note's "Generalized Delta rule" section).  Catches a wrong sign of the
    rank-one term or applying it to the updated state."""
    rng = np.random.default_rng(3)
    B, T, H, D = 2, 17, 2, 64
    _, _, _, v, _, _, S0 = _rand_inputs(rng, B, T, H, D)
    x = rng.standard_normal((B, T, H, D))
    kappa = x / np.linalg.norm(x, axis=-1, keepdims=True)
    w_log = np.full_like(x, -np.inf)
    y, sT = oracle_mod.forward(kappa, w_log, kappa, v, -kappa, kappa, S0)
    np.testing.assert_allclose(y, v, rtol=0, atol=1e-12)
    for n in range(B):
        for h in range(H):
            np.testing.assert_allclose(sT[n, h] @ kappa[n, -1, h], v[n, -1, h], rtol=0, atol=1e-12)


def _brute(r, w_log, k, v, a, b, S0):
    """S_T = S0 G_1..G_T + sum_i v_i k_i^T G_{i+1}..G_T with G_t = diag(w_t) + a_t b_t^T,
    evaluated by materialising the transition matrices (a different order of
    operations from the recurrence)."""
    T, D = r.shape
    w = np.exp(-np.exp(w_log))
    G = [np.diag(w[t]) + np.outer(a[t], b[t]) for t in range(T)]
    ys, states = [], []
    for t in range(T):
        P = np.eye(D)
        for s in range(t + 1):
            P = P @ G[s]
        S = S0 @ P
        for i in range(t + 1):
            Q = np.eye(D)
            for s in range(i + 1, t + 1):
                Q = Q @ G[s]
            S = S + np.outer(v[i], k[i]) @ Q
        states.append(S)
        ys.append(S @ r[t])
    return np.array(ys), states[-1]


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_brute_force_transition_products(oracle_mod, T):
    """General inputs, T <= 8: agreement with the materialised matrix products."""
    rng = np.random.default_rng(10 + T)
    B, H, D = 1, 2, 64
    r, w_log, k, v, a, b, S0 = _rand_inputs(rng, B, T, H, D)
    y, sT = oracle_mod.forward(r, w_log, k, v, a, b, S0)
    for h in range(H):
        Y, S = _brute(r[0, :, h], w_log[0, :, h], k[0, :, h], v[0, :, h], a[0, :, h], b[0, :, h], S0[0, h])
        np.testing.assert_allclose(y[0, :, h], Y, rtol=0, atol=1e-11)
        np.testing.assert_allclose(sT[0, h], S, rtol=0, atol=1e-11)


def test_reflections_preserve_norm(oracle_mod):
    """v = k = 0, w = 1, a = -kappa, b = 2 kappa: G = I - 2 kappa kappa^T is a
    reflection (orthogonal), so ||S_T||_F = ||S0||_F (state tracking by
    reflections, the RWKV-7 note's expressivity section)."""
    rng = np.random.default_rng(4)
    B, T, H, D = 1, 40, 2, 64
    x = rng.standard_normal((B, T, H, D))
    kappa = x / np.linalg.norm(x, axis=-1, keepdims=True)
    S0 = rng.standard_normal((B, H, D, D))
    zeros = np.zeros_like(x)
    _, sT = oracle_mod.forward(x, np.full_like(x, -np.inf), zeros, zeros, -kappa, 2 * kappa, S0)
    for h in range(H):
        assert abs(np.linalg.norm(sT[0, h]) - np.linalg.norm(S0[0, h])) < 1e-10
        # and S_T = S0 (G_1 ... G_T) is an orthogonal transform of S0's rows
        Q = np.linalg.solve(S0[0, h], sT[0, h])
        np.testing.assert_allclose(Q @ Q.T, np.eye(D), rtol=0, atol=1e-8)


def _read_fixture(name):
    rows = {}
    steps = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("step "):
                steps.append([int(x) for x in line.split()[1:]])
                continue
            key, _, rest = line.partition(":") if ":" in line else line.partition(" ")
            rows[key.strip()] = [float(x) for x in rest.split()]
    return rows, steps


def test_s5_word_fixture(oracle_mod):
    """Hand-derived permutation of the first five key columns (tests/golden/s5_transpositions.txt)."""
    rows, steps = _read_fixture("s5_transpositions.txt")
    final = [int(x) for x in rows["final"]]
    D, T = 8, len(steps)
    rng = np.random.default_rng(5)
    S0 = rng.standard_normal((1, 1, D, D))
    a = np.zeros((1, T, 1, D))
    b = np.zeros((1, T, 1, D))
    for t, (p, q) in enumerate(steps):
        a[0, t, 0, p], a[0, t, 0, q] = -1.0, 1.0
        b[0, t, 0, p], b[0, t, 0, q] = 1.0, -1.0
    zeros = np.zeros((1, T, 1, D))
    r = rng.standard_normal((1, T, 1, D))
    y, sT = oracle_mod.forward(r, np.full_like(zeros, -np.inf), zeros, zeros, a, b, S0)
    expect = S0[0, 0].copy()
    expect[:, :5] = S0[0, 0][:, final]
    # each swap evaluates s_p + (s_q - s_p): exact up to one rounding per step
    np.testing.assert_allclose(sT[0, 0], expect, rtol=0, atol=1e-13)
    np.testing.assert_allclose(y[0, -1, 0], expect @ r[0, -1, 0], rtol=0, atol=1e-12)


def test_worked_example_fixture(oracle_mod):
    """Hand-computed D = 2, T = 2 example with w = 1/2 (tests/golden/worked_example_d2.txt)."""
    rows, _ = _read_fixture("worked_example_d2.txt")
    D = 2
    S0 = np.array(rows["s0"]).reshape(1, 1, D, D)
    get = lambda n: np.stack([np.array(rows[f"t1_{n}"]), np.array(rows[f"t2_{n}"])])[None, :, None, :]
    w_log = np.full((1, 2, 1, D), np.log(np.log(2.0)))
    y, sT = oracle_mod.forward(get("r"), w_log, get("k"), get("v"), get("a"), get("b"), S0)
    np.testing.assert_allclose(y[0, 0, 0], rows["y1"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(y[0, 1, 0], rows["y2"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(sT[0, 0].ravel(), rows["sT"], rtol=0, atol=1e-12)


def test_padding_is_identity(oracle_mod):
    """l = -inf and k = v = a = b = 0 leave the state bit-for-bit unchanged and
    the output is S0 r (the padding convention of the packed batches)."""
    rng = np.random.default_rng(6)
    B, T, H, D = 2, 9, 2, 64
    r = rng.standard_normal((B, T, H, D))
    S0 = rng.standard_normal((B, H, D, D))
    zeros = np.zeros_like(r)
    y, sT = oracle_mod.forward(r, np.full_like(r, -np.inf), zeros, zeros, zeros, zeros, S0)
    np.testing.assert_array_equal(sT, S0)
    for n in range(B):
        for h in range(H):
            np.testing.assert_allclose(y[n, :, h], r[n, :, h] @ S0[n, h].T, rtol=0, atol=1e-12)


def test_chaining_is_exact(oracle_mod):
    """Constant-size state: running T1 tokens, then T2 tokens from the returned
    state, equals one run over T1 + T2 tokens, bit for bit."""
    rng = np.random.default_rng(7)
    B, T, H, D = 2, 30, 2, 64
    args = _rand_inputs(rng, B, T, H, D)
    r, w_log, k, v, a, b, S0 = args
    y, sT = oracle_mod.forward(r, w_log, k, v, a, b, S0)
    T1 = 13
    y1, s1 = oracle_mod.forward(*(x[:, :T1] for x in (r, w_log, k, v, a, b)), S0)
    y2, s2 = oracle_mod.forward(*(x[:, T1:] for x in (r, w_log, k, v, a, b)), s1)
    np.testing.assert_array_equal(np.concatenate([y1, y2], axis=1), y)
    np.testing.assert_array_equal(s2, sT)


def test_packed_equals_dense(oracle_mod):
    """A packed batch with offsets equals independent dense runs per sequence."""
    rng = np.random.default_rng(8)
    H, D = 2, 64
    lens = [5, 0, 11, 3]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(offs[-1])
    r, w_log, k, v, a, b, _ = _rand_inputs(rng, 1, Tt, H, D, s0=False)
    S0 = rng.standard_normal((len(lens), H, D, D))
    flat = [x[0] for x in (r, w_log, k, v, a, b)]
    y, sT = oracle_mod.forward(*flat, S0, seq_offsets=offs)
    for n, L in enumerate(lens):
        sl = slice(offs[n], offs[n + 1])
        yn, sn = oracle_mod.forward(*(x[None, sl] for x in flat), S0[n: n + 1])
        np.testing.assert_array_equal(y[sl], yn[0])
        np.testing.assert_array_equal(sT[n], sn[0])


def test_decode_matches_prefill(oracle_mod):
    """T decode steps with the state carried equal one T-token prefill."""
    rng = np.random.default_rng(9)
    B, T, H, D = 3, 6, 2, 64
    r, w_log, k, v, a, b, S0 = _rand_inputs(rng, B, T, H, D)
    y, sT = oracle_mod.forward(r, w_log, k, v, a, b, S0)
    s = S0
    for t in range(T):
        yt, s = oracle_mod.decode_step(*(x[:, t] for x in (r, w_log, k, v, a, b)), s)
        np.testing.assert_array_equal(yt, y[:, t])
    np.testing.assert_array_equal(s, sT)


def test_threads_do_not_change_results(oracle_mod):
    rng = np.random.default_rng(11)
    args = _rand_inputs(rng, 2, 20, 3, 64)
    y1, s1 = oracle_mod.forward(*args, n_threads=1)
    y4, s4 = oracle_mod.forward(*args, n_threads=4)
    np.testing.assert_array_equal(y1, y4)
    np.testing.assert_array_equal(s1, s4)


def test_invalid_arguments_rejected(oracle_mod):
    rng = np.random.default_rng(12)
    r, w_log, k, v, a, b, _ = _rand_inputs(rng, 1, 4, 1, 8, s0=False)
    flat = [x[0] for x in (r, w_log, k, v, a, b)]
    with pytest.raises(RuntimeError):
        oracle_mod.forward(*flat, None, seq_offsets=np.array([0, 5], dtype=np.int32))
    with pytest.raises(RuntimeError):
        oracle_mod.forward(*flat, None, seq_offsets=np.array([0, 3, 2, 4], dtype=np.int32))


def test_gated_readout_first_token_closed_form(oracle_mod):
    """Gated read-out at the first token from a zero state: S_1 = v_1 k_1^T, so
    y_1 = v_1 (k_1 . r_1) and z_1 = (v_1 (k_1 . r_1) / sqrt(D) + (sum_d r k rk) v_1) g_1.
    Written from the closed form, not from the oracle's y; catches a missing
    1/sqrt(D), an rk indexed by the wrong head, or the gate applied to one term
    only."""
    rng = np.random.default_rng(21)
    B, T, H, D = 3, 1, 4, 64
    r, w_log, k, v, a, b, _ = _rand_inputs(rng, B, T, H, D)
    rk = rng.standard_normal((H, D))
    g = rng.standard_normal((B, T, H, D))
    z, _ = oracle_mod.forward_gated(r, w_log, k, v, a, b, rk, g)
    kr = (k * r).sum(-1, keepdims=True)
    u = (r * k * rk[None, None]).sum(-1, keepdims=True)
    np.testing.assert_allclose(z, (v * kr / np.sqrt(D) + u * v) * g, rtol=0, atol=1e-12)


def test_gated_readout_special_cases(oracle_mod):
    """rk = 0 and g = 1 leave z = y / sqrt(D) (a plain rescaling of the
    recurrence output); g = 0 gives z = 0 exactly."""
    rng = np.random.default_rng(22)
    B, T, H, D = 2, 9, 2, 64
    r, w_log, k, v, a, b, S0 = _rand_inputs(rng, B, T, H, D)
    y, _ = oracle_mod.forward(r, w_log, k, v, a, b, S0)
    z, _ = oracle_mod.forward_gated(r, w_log, k, v, a, b, np.zeros((H, D)), np.ones_like(r), S0)
    np.testing.assert_allclose(z, y / 8.0, rtol=1e-15, atol=0)
    z0, _ = oracle_mod.forward_gated(r, w_log, k, v, a, b, rng.standard_normal((H, D)), np.zeros_like(r), S0)
    assert np.all(z0 == 0.0)


def _fused_inputs(rng, B, T, H, H_kv, D):
    r = rng.standard_normal((B, T, H, D))
    k, v = (rng.standard_normal((B, T, H_kv, D)) for _ in range(2))
    a_lr = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, D))))
    w_log = -np.log1p(np.exp(-rng.standard_normal((B, T, H, D)))) - 0.5
    return r, w_log, k, v, a_lr


def test_prologue_full_removal_writes_value_at_normalised_key(oracle_mod):
    """a_lr = 1 and w = 1 (l = -inf) make the step S <- S (I - kk kk^T) + v k^T with
    kk = k / ||k||: a delta-rule write with unit learning rate, after which
    S kk = ||k|| v whatever S was.  Checked step by step from random states with
    H_kv < H; catches an unnormalised or squared-norm kk, a = +kk, b without
    a_lr, or the key scaled by (1 - w) alone."""
    rng = np.random.default_rng(31)
    B, H, H_kv, D = 3, 4, 2, 64
    s = rng.standard_normal((B, H, D, D)) * 0.5
    for step in range(5):
        r, _, k, v, _ = (x[:, 0] for x in _fused_inputs(rng, B, 1, H, H_kv, D))
        w_log = np.full((B, H, D), -np.inf)
        a_lr = np.ones((B, H, D))
        _, s = oracle_mod.decode_step_fused(r, w_log, k, v, a_lr, s)
        for h in range(H):
            kh, vh = k[:, h // 2], v[:, h // 2]
            nrm = np.linalg.norm(kh, axis=-1)
            got = np.einsum("bij,bj->bi", s[:, h], kh / nrm[:, None])
            np.testing.assert_allclose(got, nrm[:, None] * vh, rtol=0, atol=1e-10)


def test_prologue_no_removal_is_a_decayed_sum(oracle_mod):
    """a_lr = 0 removes the rank-one term and scales the key by (1 - w): with a
    per-channel decay constant over time and a zero start,
    S_T[i, j] = sum_t v_t[i] k_t[j] (1 - w_j) w_j^(T-1-t).  The kv heads are
    repeated with numpy.repeat; catches a wrong (1 - w + a_lr) factor or the
    decay applied to the new token's own write."""
    rng = np.random.default_rng(32)
    B, T, H, H_kv, D = 2, 7, 4, 2, 64
    r, _, k, v, _ = _fused_inputs(rng, B, T, H, H_kv, D)
    wl_h = -np.log1p(np.exp(-rng.standard_normal((H, D)))) - 0.5
    w_log = np.broadcast_to(wl_h, (B, T, H, D)).copy()
    a_lr = np.zeros((B, T, H, D))
    _, sT = oracle_mod.forward_fused(r, w_log, k, v, a_lr)
    w = np.exp(-np.exp(wl_h))
    kr, vr = np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2)
    pw = np.stack([w ** (T - 1 - t) for t in range(T)])  # [T, H, D]
    expect = np.einsum("bthi,bthj,hj,thj->bhij", vr, kr, 1.0 - w, pw)
    np.testing.assert_allclose(sT, expect, rtol=1e-12, atol=1e-12)


def test_prologue_kv_heads_match_explicit_repeat(oracle_mod):
    """H_kv = H / 4 kv heads give exactly the result of the same inputs with
    each kv head repeated for its 4 query heads (numpy.repeat, the listing's
    repeat of k/v heads); catches a kv index of h % H_kv instead of h // 4.
    Also on the gated read-out, which must use the prologue's scaled key."""
    rng = np.random.default_rng(33)
    B, T, H, H_kv, D = 2, 9, 8, 2, 64
    r, w_log, k, v, a_lr = _fused_inputs(rng, B, T, H, H_kv, D)
    s0 = rng.standard_normal((B, H, D, D)) * 0.2
    rk = rng.standard_normal((H, D))
    g = rng.standard_normal((B, T, H, D))
    y1, s1 = oracle_mod.forward_fused(r, w_log, k, v, a_lr, s0)
    y2, s2 = oracle_mod.forward_fused(r, w_log, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2), a_lr, s0)
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(s1, s2)
    z1, _ = oracle_mod.forward_fused(r, w_log, k, v, a_lr, s0, rk=rk, g=g)
    z2, _ = oracle_mod.forward_fused(r, w_log, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2), a_lr, s0, rk=rk, g=g)
    np.testing.assert_array_equal(z1, z2)


def test_prologue_gate_uses_scaled_key(oracle_mod):
    """w = 1 and a_lr = 0 scale the key to k (1 - 1 + 0) = 0, so nothing is
    written, the state stays S0, y_t = S0 r_t and the r-k-rk term vanishes:
    z_t = (S0 r_t / sqrt(D)) g_t.  Catches the read-out using the raw key."""
    rng = np.random.default_rng(34)
    B, T, H, H_kv, D = 2, 5, 2, 1, 64
    r, _, k, v, _ = _fused_inputs(rng, B, T, H, H_kv, D)
    w_log = np.full((B, T, H, D), -np.inf)
    a_lr = np.zeros((B, T, H, D))
    s0 = rng.standard_normal((B, H, D, D)) * 0.3
    rk = rng.standard_normal((H, D))
    g = rng.standard_normal((B, T, H, D))
    z, sT = oracle_mod.forward_fused(r, w_log, k, v, a_lr, s0, rk=rk, g=g)
    np.testing.assert_array_equal(sT, s0)
    y = np.einsum("bhij,bthj->bthi", s0, r)
    np.testing.assert_allclose(z, y / np.sqrt(D) * g, rtol=1e-13, atol=1e-13)


def test_prologue_zero_key_is_identity_step(oracle_mod):
    """A zero key row (a pad token) normalises to kk = 0 (the 1e-12 floor on the
    norm, no division by zero), so with v = 0 and w = 1 the step leaves the state
    unchanged."""
    rng = np.random.default_rng(35)
    B, H, D = 2, 2, 64
    s = rng.standard_normal((B, H, D, D))
    r = rng.standard_normal((B, H, D))
    zero = np.zeros((B, 1, D))
    a_lr = rng.uniform(0.1, 0.9, (B, H, D))
    y, s1 = oracle_mod.decode_step_fused(r, np.full((B, H, D), -np.inf), zero, zero, a_lr, s)
    np.testing.assert_array_equal(s1, s)
    assert np.all(np.isfinite(y))


def _bwd_loss(oracle_mod, args, dy, dsT, offs=None):
    y, sT = oracle_mod.forward(*args, seq_offsets=offs)
    return float(np.sum(y * dy) + np.sum(sT * dsT))


@pytest.mark.parametrize("packed", [False, True])
def test_backward_matches_finite_differences(oracle_mod, packed):
    """The backward's gradients of L = <dy, y> + <dsT, sT> against central
    differences of the (separately pinned) forward along random directions, for
    every input: r, w_log, k, v, a, b and s0.  fp64 with eps = 1e-6 leaves a
    truncation and rounding error near 1e-9, so a dropped term, a wrong sign or
    a transposed product fails by orders of magnitude."""
    rng = np.random.default_rng(41 + packed)
    B, T, H, D = 2, 7, 2, 64
    r, w_log, k, v, a, b, S0 = _rand_inputs(rng, B, T, H, D)
    dy = rng.standard_normal((B, T, H, D))
    dsT = rng.standard_normal((B, H, D, D))
    offs = None
    if packed:
        # sequences of 3 and 11 tokens on one packed axis
        flat = lambda x: x.reshape(B * T, H, D)
        r, w_log, k, v, a, b, dy = (flat(x).copy() for x in (r, w_log, k, v, a, b, dy))
        offs = np.array([0, 3, 14], dtype=np.int32)
    args = [r, w_log, k, v, a, b, S0]
    grads = oracle_mod.backward(r, w_log, k, v, a, b, dy, S0, dsT, offs)
    eps = 1e-6
    for idx, X in enumerate(args):
        for _ in range(2):
            u = rng.standard_normal(X.shape)
            plus = list(args)
            minus = list(args)
            plus[idx] = X + eps * u
            minus[idx] = X - eps * u
            fd = (_bwd_loss(oracle_mod, plus, dy, dsT, offs) - _bwd_loss(oracle_mod, minus, dy, dsT, offs)) / (2 * eps)
            an = float(np.sum(grads[idx] * u))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, fd, an)


def test_backward_linear_attention_closed_form(oracle_mod):
    """a = b = 0 and w = 1 (l = -inf): y_t = S0 r_t + sum_{s<=t} (k_s . r_t) v_s, so
    dv_s = sum_{t>=s} (r_t . k_s) dy_t + dsT k_s, dk_s = sum_{t>=s} (v_s . dy_t) r_t +
    dsT^T v_s, dr_t = S_t^T dy_t, ds0 = sum_t dy_t r_t^T + dsT, and the decay logit,
    a and b get the gradients of their linear terms.  Written with numpy from
    this closed form."""
    rng = np.random.default_rng(43)
    B, T, H, D = 1, 6, 1, 64
    r, _, k, v, _, _, S0 = _rand_inputs(rng, B, T, H, D)
    zero = np.zeros((B, T, H, D))
    w_log = np.full((B, T, H, D), -np.inf)
    dy = rng.standard_normal((B, T, H, D))
    dsT = rng.standard_normal((B, H, D, D))
    dr, dwl, dk, dv, da, db, ds0 = oracle_mod.backward(r, w_log, k, v, zero, zero, dy, S0, dsT)
    R, K, V, DY = (x[0, :, 0] for x in (r, k, v, dy))
    mask = np.triu(np.ones((T, T)))  # mask[s, t] = 1 for t >= s
    RK = (K @ R.T) * mask            # RK[s, t] = k_s . r_t for t >= s
    VD = (V @ DY.T) * mask           # VD[s, t] = v_s . dy_t for t >= s
    exp_dv = RK @ DY + K @ dsT[0, 0].T
    exp_dk = VD @ R + V @ dsT[0, 0]
    S = S0[0, 0] + np.cumsum(np.einsum("ti,tj->tij", V, K), axis=0)
    exp_dr = np.einsum("tij,ti->tj", S, DY)
    exp_ds0 = DY.T @ R + dsT[0, 0]
    np.testing.assert_allclose(dv[0, :, 0], exp_dv, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(dk[0, :, 0], exp_dk, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(dr[0, :, 0], exp_dr, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(ds0[0, 0], exp_ds0, rtol=1e-10, atol=1e-10)
    assert np.all(dwl == 0.0)  # w = 1 exactly: dw/dl = -exp(l) w = 0


# ------------------------------------------------------------------ state maps (sequence split)
@pytest.mark.parametrize("T", [1, 3, 8])
def test_state_map_is_the_transition_product(oracle_mod, T):
    """M = G_1 G_2 ... G_T with G_t = diag(w_t) + a_t b_t^T materialised as
    matrices, and Q = the brute-force end state from a zero start (catches a
    reversed product order, a dropped rank-one term, or v leaking into M)."""
    rng = np.random.default_rng(40 + T)
    B, H, D = 1, 2, 64
    r, w_log, k, v, a, b, _ = _rand_inputs(rng, B, T, H, D, s0=False)
    M, Q = oracle_mod.state_map(w_log, k, v, a, b)
    w = np.exp(-np.exp(w_log))
    for h in range(H):
        P = np.eye(D)
        for t in range(T):
            P = P @ (np.diag(w[0, t, h]) + np.outer(a[0, t, h], b[0, t, h]))
        np.testing.assert_allclose(M[0, h], P, rtol=0, atol=1e-12)
        _, S = _brute(r[0, :, h], w_log[0, :, h], k[0, :, h], v[0, :, h], a[0, :, h], b[0, :, h], np.zeros((D, D)))
        np.testing.assert_allclose(Q[0, h], S, rtol=0, atol=1e-12)


def test_state_map_gives_every_end_state(oracle_mod):
    """For any start state S0 the recurrence ends at S0 M + Q (dense batch and
    a packed batch with pads and an empty sequence)."""
    rng = np.random.default_rng(50)
    B, T, H, D = 2, 150, 2, 64
    r, w_log, k, v, a, b, S0 = _rand_inputs(rng, B, T, H, D)
    M, Q = oracle_mod.state_map(w_log, k, v, a, b)
    _, sT = oracle_mod.forward(r, w_log, k, v, a, b, S0)
    np.testing.assert_allclose(sT, S0 @ M + Q, rtol=0, atol=1e-10)
    offs = np.array([0, 70, 70, 200], dtype=np.int32)
    r, w_log, k, v, a, b, _ = _rand_inputs(rng, 1, 200, H, D, s0=False)
    pk = [x[0] for x in (r, w_log, k, v, a, b)]
    pk[1][60:70] = -np.inf  # pad tokens: w = 1, k = v = a = b = 0
    for i in (2, 3, 4, 5):
        pk[i][60:70] = 0.0
    S0 = rng.standard_normal((3, H, D, D))
    M, Q = oracle_mod.state_map(*pk[1:], seq_offsets=offs)
    _, sT = oracle_mod.forward(*pk, S0, seq_offsets=offs)
    np.testing.assert_allclose(sT, S0 @ M + Q, rtol=0, atol=1e-10)
    np.testing.assert_array_equal(M[1], np.broadcast_to(np.eye(D), (H, D, D)))  # empty sequence: identity
    np.testing.assert_array_equal(Q[1], 0.0)


def test_state_maps_compose_over_ranges(oracle_mod):
    """The map of [0, T) is the composition of the maps of [0, T1) and [T1, T):
    M = M1 M2 and Q = Q1 M2 + Q2 (the exclusive scan of a sequence split)."""
    rng = np.random.default_rng(51)
    B, T, H, D = 1, 130, 2, 64
    r, w_log, k, v, a, b, _ = _rand_inputs(rng, B, T, H, D, s0=False)
    T1 = 64
    M, Q = oracle_mod.state_map(w_log, k, v, a, b)
    M1, Q1 = oracle_mod.state_map(*(x[:, :T1] for x in (w_log, k, v, a, b)))
    M2, Q2 = oracle_mod.state_map(*(x[:, T1:] for x in (w_log, k, v, a, b)))
    np.testing.assert_allclose(M, M1 @ M2, rtol=0, atol=1e-11)
    np.testing.assert_allclose(Q, Q1 @ M2 + Q2, rtol=0, atol=1e-11)
