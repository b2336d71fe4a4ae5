"""Pins of the CPU oracle to what the pages and the mathematics fix (no GPU).

Each test ties one oracle function to something other than itself: a value the
pages print (tests/golden), a closed form, a special case that reduces to a
textbook/library computation, or brute force on tiny inputs.  Each is chosen so
that a plausible mistake (a dropped term, a wrong sign or index, a transposed
operand, a wrong claim order) fails it.
"""
import itertools
import math

import numpy as np
import pytest

import oracle


# ---------------------------------------------------------------- router ----

def _router_for_logits(x, logits):
    """A W_r (rows = experts) with W_r x = logits for the given x, built with a
    non-trivial dependence on every input coordinate."""
    x = np.asarray(x, np.float64)
    N, d = len(logits), len(x)
    rng = np.random.default_rng(7)
    w = rng.choice([-0.5, 0.25, 0.5], size=(N, d)).astype(np.float64)
    j = int(np.argmax(np.abs(x)))
    for i in range(N):
        rest = w[i] @ x - w[i, j] * x[j]
        w[i, j] = (logits[i] - rest) / x[j]
    return w.astype(np.float32)


def test_worked_top2_gating_example(golden):
    g = golden("gating_worked_example.txt")
    x = np.array([g["x"]], np.float32)
    w_r = _router_for_logits(g["x"], g["logits"])
    r = oracle.route(x, w_r, None, k=g["k"])
    np.testing.assert_allclose(r["logits"][0], g["logits"], atol=1e-6)
    G = np.zeros(len(g["logits"]))
    G[r["idx"][0]] = r["gate"][0]
    np.testing.assert_array_equal(np.round(G, g["decimals"]), np.array(g["G"], float))
    assert list(r["idx"][0]) == [1, 0] or list(r["idx"][0]) == [0, 1]
    assert r["idx"][0, 0] == 1  # 1.6 is the largest logit


def test_softmax_init_examples(golden):
    g = golden("softmax_init_examples.txt")
    for lk, pk in (("logits_s1", "probs_s1"), ("logits_s01", "probs_s01")):
        logits = g[lk]
        x = np.array([[1.0, 0.0]], np.float32)
        w_r = np.array([[v, 0.0] for v in logits], np.float32)
        r = oracle.route(x, w_r, None, k=1)
        np.testing.assert_array_equal(np.round(r["probs"][0].astype(np.float64), g["decimals"]),
                                      np.array(g[pk], float))


def test_softmax_closed_form_ratios():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((16, 24)).astype(np.float32)
    w = rng.standard_normal((6, 24)).astype(np.float32) * 0.3
    r = oracle.route(x, w, None, k=1)
    p = r["probs"].astype(np.float64)
    h = r["logits"].astype(np.float64)
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-6)
    # p_i / p_0 = exp(h_i - h_0): pins the sign and the operand of the exponent
    np.testing.assert_allclose(p / p[:, :1], np.exp(h - h[:, :1]), rtol=2e-6)
    # logits are the row dot products x W_r^T (a transposed W_r fails here)
    np.testing.assert_allclose(h, x.astype(np.float64) @ w.astype(np.float64).T, rtol=1e-6, atol=1e-6)


def test_gate_topk_renormalisation_identity():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 32)).astype(np.float32)
    w = rng.standard_normal((8, 32)).astype(np.float32) * 0.2
    r1 = oracle.route(x, w, None, k=1)
    r2 = oracle.route(x, w, None, k=2)
    p = r1["probs"].astype(np.float64)
    # top-1: the gate is the full-softmax probability of the argmax
    np.testing.assert_allclose(r1["gate"][:, 0], p[np.arange(64), r1["idx"][:, 0]], rtol=1e-6)
    np.testing.assert_array_equal(r1["idx"][:, 0], np.argmax(r1["logits"], axis=1))
    # top-2: the second choice is the argmax of the rest; gates = p_i / (p_i1 + p_i2)
    np.testing.assert_array_equal(r2["idx"][:, 0], r1["idx"][:, 0])
    masked = r1["logits"].astype(np.float64).copy()
    masked[np.arange(64), r1["idx"][:, 0]] = -np.inf
    np.testing.assert_array_equal(r2["idx"][:, 1], np.argmax(masked, axis=1))
    pi = p[np.arange(64)[:, None], r2["idx"]]
    np.testing.assert_allclose(r2["gate"], pi / pi.sum(1, keepdims=True), rtol=2e-6)
    np.testing.assert_allclose(r2["gate"].sum(1), 1.0, rtol=1e-6)
    assert np.all(r2["gate"][:, 0] >= r2["gate"][:, 1])


def test_zero_router_ties_go_to_lowest_indices():
    # CMU 10-423 Lecture 16 section 2.3: an all-zero router gives equal logits and
    # top-k always picks the smallest indices.
    T, N = 40, 8
    x = np.random.default_rng(3).standard_normal((T, 16)).astype(np.float32)
    w = np.zeros((N, 16), np.float32)
    r1 = oracle.route(x, w, None, k=1)
    r2 = oracle.route(x, w, None, k=2)
    assert np.all(r1["idx"][:, 0] == 0)
    assert np.all(r2["idx"][:, 0] == 0) and np.all(r2["idx"][:, 1] == 1)
    np.testing.assert_array_equal(r1["probs"], np.full((T, N), 1.0 / N, np.float32))
    f, P, aux = oracle.aux_loss(r1["idx"], r1["probs"], alpha=1e-2)
    np.testing.assert_array_equal(f, [1.0] + [0.0] * (N - 1))
    assert aux == pytest.approx(1e-2, rel=1e-15)
    d = oracle.dispatch(r2["idx"], N, C=T)
    np.testing.assert_array_equal(d["counts"][0], [T] + [0] * (N - 1))
    np.testing.assert_array_equal(d["counts"][1], [0, T] + [0] * (N - 2))


def test_bf16_rounding_and_fp32_router(golden):
    g = golden("bf16_rounding_example.txt")
    assert oracle.bf16_round(g["logit_e0"]) == np.float32(g["bf16_e0"])
    assert oracle.bf16_round(g["logit_e1"]) == np.float32(g["bf16_e1"])
    # spacing of bf16 in [4, 8): the next value after 4.0
    nxt = oracle.widen(np.array([oracle.bf16_bits(4.0) + 1], np.uint16))[0]
    assert nxt - 4.0 == g["bf16_spacing_4_8"]
    # the fp32 router still separates them
    x = np.array([[1.0]], np.float32)
    w = np.array([[g["logit_e0"]], [g["logit_e1"]]], np.float32)
    assert oracle.route(x, w, None, k=1)["idx"][0, 0] == g["fp32_winner"]
    # round-to-nearest-even on exact ties, and carry into the exponent
    assert oracle.bf16_round(1.0 + 2.0 ** -8) == np.float32(1.0)          # tie, even stays
    assert oracle.bf16_round(1.0 + 3 * 2.0 ** -8) == np.float32(1.0 + 2.0 ** -6)  # tie, odd rounds up
    assert oracle.bf16_round(np.nextafter(np.float32(2.0), np.float32(0))) == np.float32(2.0)
    assert oracle.bf16_round(-4.01) == np.float32(-4.0)


def test_router_bias_is_added():
    x = np.array([[1.0, 2.0]], np.float32)
    w = np.array([[0.5, 0.0], [0.0, 0.25]], np.float32)
    r = oracle.route(x, w, np.array([0.0, 0.1], np.float32), k=1)
    np.testing.assert_allclose(r["logits"][0], [0.5, 0.6], rtol=1e-6)
    assert r["idx"][0, 0] == 1


# ------------------------------------------------------------- aux loss -----

def test_aux_equals_alpha_under_uniform_f():
    # one-hot dominant logits in a round-robin: each expert is the top-1 of T/N tokens
    N, m = 8, 5
    T = N * m
    x = np.zeros((T, N), np.float32)
    for t in range(T):
        x[t, t % N] = 2.0 + 0.5 * (t % N)   # experts differ in how peaked they are
        x[t, (t + 3) % N] = 1.0
    w = np.eye(N, dtype=np.float32)
    r = oracle.route(x, w, None, k=1)
    f, P, aux = oracle.aux_loss(r["idx"], r["probs"], alpha=1e-2)
    np.testing.assert_allclose(f, 1.0 / N, rtol=0, atol=0)
    assert aux == pytest.approx(1e-2, rel=1e-7)      # alpha * N * sum (1/N) P_i = alpha
    assert np.max(P) - np.min(P) > 0.05              # P itself is not uniform


def test_aux_counts_top1_only_and_cauchy_schwarz():
    T, N = 64, 4
    x = np.zeros((T, N), np.float32)
    for t in range(T):
        x[t, 0] = 4.0
        x[t, 1 + t % 3] = 2.0
    r = oracle.route(x, np.eye(N, dtype=np.float32), None, k=2)
    f, P, aux = oracle.aux_loss(r["idx"], r["probs"], alpha=0.5)
    np.testing.assert_array_equal(f, [1.0, 0.0, 0.0, 0.0])   # column 0 only
    assert aux == pytest.approx(0.5 * N * P[0], rel=1e-12)
    # when P == f the loss is alpha N sum f^2 >= alpha (Cauchy-Schwarz), equality iff uniform
    for fv in ([0.25] * 4, [0.7, 0.1, 0.1, 0.1], [1.0, 0, 0, 0]):
        fv = np.array(fv)
        assert 0.5 * N * float(fv @ fv) >= 0.5 - 1e-15


def test_aux_empty_batch():
    f, P, aux = oracle.aux_loss(np.zeros((0, 1), np.int32), np.zeros((0, 4), np.float32))
    assert aux == 0.0 and not f.any() and not P.any()


# ------------------------------------------------------------- capacity -----

# ---------------------------------------------------------------- z-loss ----

def test_z_loss_uniform_router_closed_form():
    # equal logits c on N experts: log sum exp = c + ln N for every token
    for N, c in [(1, 0.0), (8, 0.0), (64, 0.0), (8, 1.5), (128, -3.25)]:
        logits = np.full((5, N), c, np.float32)
        assert oracle.z_loss(logits) == pytest.approx((c + math.log(N)) ** 2, rel=1e-15, abs=1e-15)


def test_z_loss_matches_library_logsumexp():
    from scipy.special import logsumexp
    rng = np.random.default_rng(3)
    logits = (rng.standard_normal((37, 11)) * 4.0).astype(np.float32)
    want = np.mean(logsumexp(logits.astype(np.float64), axis=1) ** 2)
    assert oracle.z_loss(logits) == pytest.approx(want, rel=1e-13)


def test_z_loss_large_logits_and_shift():
    # max-shifted evaluation: huge logits do not overflow; a shift by c moves
    # every token's log-sum-exp by c; permuting experts changes nothing
    logits = np.array([[1000.0, 999.0, -5.0], [-1000.0, -1000.0, -1000.0]], np.float32)
    l0 = 1000.0 + math.log(1.0 + math.exp(-1.0) + math.exp(-1005.0))
    l1 = -1000.0 + math.log(3.0)
    assert oracle.z_loss(logits) == pytest.approx((l0 * l0 + l1 * l1) / 2, rel=1e-14)
    # one token at a time, logits >= 4 so every log-sum-exp is positive:
    # sqrt(z) is the log-sum-exp, and a shift by c adds c to it
    rng = np.random.default_rng(5)
    h = (4.0 + rng.random((9, 6))).astype(np.float32)
    c = np.float32(2.0)
    for t in range(9):
        one = h[t:t + 1]
        assert math.sqrt(oracle.z_loss(one + c)) == pytest.approx(math.sqrt(oracle.z_loss(one)) + 2.0, rel=1e-12)
    assert oracle.z_loss(h[:, ::-1].copy()) == pytest.approx(oracle.z_loss(h), rel=1e-14)


def test_z_loss_empty_batch():
    assert oracle.z_loss(np.zeros((0, 4), np.float32)) == 0.0


def test_capacity_exercise(golden):
    g = golden("capacity_exercise.txt")
    C = oracle.capacity(g["T"], g["N"], g["k"], g["cf"])
    assert C == g["C"]
    T, N, k = g["T"], g["N"], g["k"]
    # (b) uniform routing: token t picks experts t mod N and (t + 1) mod N
    idx = np.stack([np.arange(T) % N, (np.arange(T) + 1) % N], 1).astype(np.int32)
    d = oracle.dispatch(idx, N, C)
    assert np.all(d["counts"].sum(0) == g["uniform_per_expert"])
    assert int(d["drop"].sum()) == g["uniform_dropped"]
    # (c) one expert receives 512 of the 2048 assignments
    idx = np.zeros((T, 2), np.int32)
    hot = g["hot_assignments"]
    idx[:hot, 0] = 0
    idx[hot:, 0] = 1 + (np.arange(T - hot) % (N - 1))
    idx[:, 1] = 1 + (np.arange(T) % (N - 1))
    idx[hot:, 1] = np.where(idx[hot:, 1] == idx[hot:, 0], 1 + (idx[hot:, 1] % (N - 1)), idx[hot:, 1])
    assert np.all(idx[:, 0] != idx[:, 1])
    per_expert = np.bincount(idx.reshape(-1), minlength=N)
    assert per_expert[0] == hot and per_expert[1:].max() <= C
    d = oracle.dispatch(idx, N, C)
    assert int(d["drop"].sum()) == g["hot_dropped"]
    assert round(100.0 * d["drop"].sum() / (k * T), 1) == g["hot_dropped_percent"]
    # the kept claims on the hot expert are its first C rank-0 tokens, in token order
    assert np.all(d["drop"][:C, 0] == 0) and np.all(d["drop"][C:hot, 0] == 1)


def test_capacity_exact_floor():
    assert oracle.capacity(65536, 64, 1, 1.25) == 1280
    assert oracle.capacity(512, 8, 1, 1.0) == 64
    assert oracle.capacity(65536, 128, 1, 1.0) == 512
    assert oracle.capacity(32768, 32, 2, 2.0) == 4096
    assert oracle.capacity(16384, 8, 2, 1.25) == 5120
    assert oracle.capacity(10, 3, 1, 1.0) == 3
    assert oracle.capacity(0, 8, 1, 1.25) == 0
    assert oracle.capacity(100, 8, 1, 0.0) == 0
    # the double 0.1 is slightly above 1/10, the double 0.3 slightly below 3/10
    assert oracle.capacity(10, 1, 1, 0.1) == 1
    assert oracle.capacity(10, 1, 1, 0.3) == 2
    assert oracle.capacity(-1, 8, 1, 1.0) == -1
    assert oracle.capacity(8, 0, 1, 1.0) == -1
    from fractions import Fraction
    rng = np.random.default_rng(5)
    for _ in range(300):
        T = int(rng.integers(0, 1 << 20)); N = int(rng.integers(1, 129)); k = int(rng.integers(1, 3))
        cf = float(rng.choice([0.5, 1.0, 1.25, 1.5, 2.0, 0.1, 0.3, 1.1, 3.7, float(rng.random() * 4)]))
        want = math.floor(Fraction(k * T) * Fraction(cf) / N)
        assert oracle.capacity(T, N, k, cf) == want


def test_idle_capacity_identity():
    # without drops the idle slot fraction is 1 - kT/(NC); at C = cf kT/N it is 1 - 1/cf
    T, N, k, cf = 256, 8, 2, 2.0
    C = oracle.capacity(T, N, k, cf)
    idx = np.stack([np.arange(T) % N, (np.arange(T) + 5) % N], 1).astype(np.int32)
    d = oracle.dispatch(idx, N, C)
    assert d["drop"].sum() == 0
    idle = 1.0 - d["kept"].sum() / (N * C)
    assert idle == pytest.approx(1.0 - 1.0 / cf, abs=1e-15)


def _literal_dispatch(idx, N, C):
    """Literal transcription of the pages' capacity loop: per expert a list of
    slots; a token is appended while the list is shorter than C, else skipped;
    all tokens' first choices are placed before any second choice."""
    T, k = idx.shape
    slots = [[] for _ in range(N)]
    kept = set()
    for r in range(k):
        for t in range(T):
            target = int(idx[t, r])
            if len(slots[target]) < C:
                slots[target].append((t, r))
                kept.add((t, r))
    return slots, kept


@pytest.mark.parametrize("k", [1, 2])
def test_dispatch_brute_force(k):
    for N in (1, 2, 3):
        if k > N:
            continue
        for T in range(0, 5 if k == 2 else 6):
            choices = [c for c in itertools.product(range(N), repeat=k) if len(set(c)) == k]
            for combo in itertools.product(choices, repeat=T):
                idx = np.array(combo, np.int32).reshape(T, k)
                for C in range(0, k * T + 2):
                    d = oracle.dispatch(idx, N, C)
                    slots, kept = _literal_dispatch(idx, N, C)
                    for e in range(N):
                        assert d["kept"][e] == len(slots[e])
                        for j, (t, r) in enumerate(slots[e]):
                            assert d["pos"][t, r] == j and d["drop"][t, r] == 0
                    for t in range(T):
                        for r in range(k):
                            assert bool(d["drop"][t, r]) == ((t, r) not in kept)
                    np.testing.assert_array_equal(
                        d["counts"].sum(0), np.bincount(idx.reshape(-1), minlength=N))
                    np.testing.assert_array_equal(d["offsets"], np.concatenate([[0], np.cumsum(d["kept"])]))


# ------------------------------------------------------- batch priority ----

def _rand_routing(T, N, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(N)[:k] for _ in range(T)]).astype(np.int32)
    gate = rng.random((T, k)).astype(np.float32)
    return idx, gate


@pytest.mark.parametrize("k", [1, 2])
def test_priority_with_equal_or_decreasing_scores_is_token_order(k):
    # equal scores (ties to the lower index) and scores decreasing in t both
    # give exactly the token-order claim, for every capacity
    T, N = 40, 5
    idx, gate = _rand_routing(T, N, k, 11)
    flat = np.full((T, k), 0.25, np.float32)
    dec = np.repeat(np.linspace(1.0, 0.1, T, dtype=np.float32)[:, None], k, axis=1)
    for C in (0, 3, 8, 40):
        ref = oracle.dispatch(idx, N, C)
        for pr in (flat, dec):
            got = oracle.dispatch(idx, N, C, priority=pr)
            for key in ref:
                np.testing.assert_array_equal(got[key], ref[key], err_msg=key)


@pytest.mark.parametrize("k", [1, 2])
def test_priority_increasing_scores_is_reversed_token_order(k):
    # scores increasing in t claim in reversed token order: the same as the
    # token-order dispatch of the reversed batch, read back reversed
    T, N = 33, 4
    idx, _ = _rand_routing(T, N, k, 12)
    inc = np.repeat(np.linspace(0.1, 1.0, T, dtype=np.float32)[:, None], k, axis=1)
    for C in (0, 2, 5, 33):
        rev = oracle.dispatch(idx[::-1].copy(), N, C)
        got = oracle.dispatch(idx, N, C, priority=inc)
        np.testing.assert_array_equal(got["pos"], rev["pos"][::-1])
        np.testing.assert_array_equal(got["drop"], rev["drop"][::-1])
        for key in ("counts", "kept", "offsets"):
            np.testing.assert_array_equal(got[key], rev[key])


def test_priority_top1_keeps_the_highest_scores_per_expert():
    # top-1: an expert keeps exactly its C claimants with the largest scores
    # (ties to the lower index), whatever their positions in the batch
    T, N, C = 200, 6, 9
    idx, gate = _rand_routing(T, N, 1, 13)
    gate[::7, 0] = gate[3, 0]                   # plant ties
    got = oracle.dispatch(idx, N, C, priority=gate)
    for e in range(N):
        ts = np.nonzero(idx[:, 0] == e)[0]
        ranked = sorted(ts, key=lambda t: (-float(gate[t, 0]), t))
        kept = set(ranked[:C])
        assert set(ts[got["drop"][ts, 0] == 0]) == kept
        for n, t in enumerate(ranked):
            assert got["pos"][t, 0] == n


# ------------------------------------------------- no token left behind ----

def _probs(T, N, seed):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((T, N))
    p = np.exp(h - h.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)).astype(np.float32)


def test_ntlb_without_overflow_is_the_top1_dispatch():
    # C >= T: nobody overflows, so stage 0 alone is the token-order top-1 claim
    T, N = 60, 5
    p = _probs(T, N, 21)
    top1 = np.argmax(p, axis=1).astype(np.int32)            # no exact ties in random data
    ref = oracle.dispatch(top1[:, None], N, T)
    got = oracle.dispatch_ntlb(p, p[np.arange(T), top1], T)
    np.testing.assert_array_equal(got["expert"], top1)
    np.testing.assert_array_equal(got["pos"], ref["pos"][:, 0])
    np.testing.assert_array_equal(got["drop"], ref["drop"][:, 0])
    np.testing.assert_array_equal(got["offsets"], ref["offsets"])
    np.testing.assert_array_equal(got["gate"], p[np.arange(T), top1])


@pytest.mark.parametrize("C", [0, 1, 4, 7, 12, 30])
def test_ntlb_drops_only_when_every_expert_is_full(C):
    T, N = 30, 4
    p = _probs(T, N, 22)
    top1 = np.argmax(p, axis=1)
    got = oracle.dispatch_ntlb(p, p[np.arange(T), top1], C)
    kept = got["kept"]
    assert int(kept.sum()) == min(T, N * C)                  # a slot left anywhere takes a token
    assert int((got["drop"] == 0).sum()) == min(T, N * C)
    assert np.all(kept <= C)
    # stage 0 keeps exactly the token-order top-1 claims below C
    ref = oracle.dispatch(top1[:, None].astype(np.int32), N, C)
    first = ref["drop"][:, 0] == 0
    np.testing.assert_array_equal(got["expert"][first], top1[first])
    np.testing.assert_array_equal(got["pos"][first], ref["pos"][first, 0])
    # a kept token's gate is its probability for the expert that kept it, and
    # every expert it prefers to that one was already full when it tried it
    for t in np.nonzero(got["drop"] == 0)[0]:
        e = got["expert"][t]
        assert got["gate"][t] == p[t, e]
        assert got["pos"][t] < C
    rows = got["offsets"][got["expert"][got["drop"] == 0]] + got["pos"][got["drop"] == 0]
    assert sorted(rows.tolist()) == list(range(int(kept.sum())))   # compact rows tile exactly


def test_ntlb_small_hand_example():
    # 3 tokens, 2 experts, C = 1.  All prefer expert 0: token 0 takes it in
    # stage 0; in stage 1 token 1 takes expert 1 and token 2 finds it full.
    p = np.array([[0.9, 0.1], [0.8, 0.2], [0.7, 0.3]], np.float32)
    got = oracle.dispatch_ntlb(p, p[:, 0], 1)
    np.testing.assert_array_equal(got["expert"], [0, 1, 0])
    np.testing.assert_array_equal(got["drop"], [0, 0, 1])
    np.testing.assert_array_equal(got["pos"], [0, 0, 1])
    np.testing.assert_array_equal(got["counts"], [3, 2])
    np.testing.assert_array_equal(got["kept"], [1, 1])
    np.testing.assert_allclose(got["gate"], [0.9, 0.2, 0.7])


# ------------------------------------------------------ router backward ----

def _fwd_loss(x, w, b, idx, f, dgate, alpha):
    """sum dgate * gate + L_aux in fp64, with the expert selection and f held
    fixed (the forward's definitions: softmax router, top-1 gate p_{i*} or the
    softmax over the two kept logits, aux = alpha N sum f_i P_i)."""
    h = x @ w.T + b
    p = np.exp(h - h.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    T, N = p.shape
    k = idx.shape[1]
    if k == 1:
        g = p[np.arange(T), idx[:, 0]][:, None]
    else:
        h1, h2 = h[np.arange(T), idx[:, 0]], h[np.arange(T), idx[:, 1]]
        g1 = 1.0 / (1.0 + np.exp(h2 - h1))
        g = np.stack([g1, 1.0 - g1], axis=1)
    return float((dgate * g).sum() + alpha * N * (f * p.mean(axis=0)).sum()), p, g


@pytest.mark.parametrize("k", [1, 2])
def test_router_backward_matches_finite_differences(k):
    rng = np.random.default_rng(40 + k)
    T, N, d, alpha = 6, 5, 4, 0.3
    x = rng.standard_normal((T, d))
    w = rng.standard_normal((N, d)) * 0.7
    b = rng.standard_normal(N) * 0.2
    h = x @ w.T + b
    idx = np.argsort(-h, axis=1, kind="stable")[:, :k].astype(np.int32)
    f = rng.random(N)
    f /= f.sum()
    dgate = rng.standard_normal((T, k))
    _, p, g = _fwd_loss(x, w, b, idx, f, dgate, alpha)
    got = oracle.router_backward(x.astype(np.float32), w.astype(np.float32), p.astype(np.float32), idx,
                                 g.astype(np.float32), f, dgate.astype(np.float32), alpha)
    # the oracle reads x and W_r as fp32: differentiate at those values
    x32, w32 = x.astype(np.float32).astype(np.float64), w.astype(np.float32).astype(np.float64)
    dg32 = dgate.astype(np.float32).astype(np.float64)

    def num_grad(fun, a, eps=1e-6):
        out = np.zeros_like(a)
        for i in np.ndindex(a.shape):
            hi, lo = a.copy(), a.copy()
            hi[i] += eps
            lo[i] -= eps
            out[i] = (fun(hi) - fun(lo)) / (2 * eps)
        return out

    L = lambda xx, ww, bb: _fwd_loss(xx, ww, bb, idx, f, dg32, alpha)[0]
    np.testing.assert_allclose(got["dw"], num_grad(lambda ww: L(x32, ww, b), w32), rtol=2e-5, atol=1e-7)
    np.testing.assert_allclose(got["db"], num_grad(lambda bb: L(x32, w32, bb), b.copy()), rtol=2e-5, atol=1e-7)
    np.testing.assert_allclose(got["dx"], num_grad(lambda xx: L(xx, w32, b), x32), rtol=2e-5, atol=1e-7)


def test_router_backward_uniform_f_has_no_aux_gradient():
    # equal f_i: dL_aux/dp_{t,i} is the same for every expert, and the softmax
    # Jacobian maps a constant vector to zero
    rng = np.random.default_rng(44)
    T, N, d = 7, 6, 5
    x = rng.standard_normal((T, d)).astype(np.float32)
    w = rng.standard_normal((N, d)).astype(np.float32)
    r = oracle.route(x, w, None, 1)
    got = oracle.router_backward(x, w, r["probs"], r["idx"], r["gate"], np.full(N, 1.0 / N), np.zeros((T, 1), np.float32),
                                 alpha=0.5)
    assert np.abs(got["dh"]).max() < 1e-7


# ------------------------------------------------------ expert backward ----

@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_expert_backward_matches_finite_differences(act):
    rng = np.random.default_rng(50 if act == "relu" else 51)
    T, d, d_ff, N, k = 4, 3, 5, 3, 2
    f32 = lambda a: np.asarray(a, np.float32)
    W = dict(w1=f32(rng.standard_normal((N, d_ff, d))), b1=f32(rng.standard_normal((N, d_ff)) * 0.3),
             w2=f32(rng.standard_normal((N, d, d_ff))), b2=f32(rng.standard_normal((N, d)) * 0.3))
    if act == "swiglu":
        W.update(w3=f32(rng.standard_normal((N, d_ff, d))), b3=f32(rng.standard_normal((N, d_ff)) * 0.3))
    x = f32(rng.standard_normal((T, d)))
    idx = np.stack([rng.permutation(N)[:k] for _ in range(T)]).astype(np.int32)
    gate = f32(rng.random((T, k)))
    drop = np.zeros((T, k), np.uint8)
    drop[1, 1] = 1                                           # a dropped assignment contributes nothing
    dout = f32(rng.standard_normal((T, d)))
    P64 = {key: v.astype(np.float64) for key, v in W.items()}

    def loss(x_, g_, P):
        L = 0.0
        for t in range(T):
            for r in range(k):
                if drop[t, r]:
                    continue
                e = idx[t, r]
                u = P["w1"][e] @ x_[t] + P["b1"][e]
                if act == "relu":
                    a = np.maximum(u, 0.0)
                else:
                    v = P["w3"][e] @ x_[t] + P["b3"][e]
                    a = u / (1.0 + np.exp(-u)) * v
                y = P["w2"][e] @ a + P["b2"][e]
                L += g_[t, r] * float(dout[t].astype(np.float64) @ y)
        return L

    if act == "relu":   # finite differences need every preactivation away from the kink
        for t in range(T):
            for r in range(k):
                u = P64["w1"][idx[t, r]] @ x[t].astype(np.float64) + P64["b1"][idx[t, r]]
                assert np.abs(u).min() > 1e-3

    def num(fun, a, eps=1e-6):
        out = np.zeros_like(a)
        for i in np.ndindex(a.shape):
            hi, lo = a.copy(), a.copy()
            hi[i] += eps
            lo[i] -= eps
            out[i] = (fun(hi) - fun(lo)) / (2 * eps)
        return out

    got = oracle.expert_backward(x, W, idx, gate, drop, dout, act=oracle.SWIGLU if act == "swiglu" else oracle.RELU)
    x64, g64 = x.astype(np.float64), gate.astype(np.float64)
    tol = dict(rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(got["dgate"], num(lambda g_: loss(x64, g_, P64), g64) * (1 - drop), **tol)
    np.testing.assert_allclose(got["dx"], num(lambda x_: loss(x_, g64, P64), x64), **tol)
    for key in W:
        ref = num(lambda a_: loss(x64, g64, {**P64, key: a_}), P64[key])
        np.testing.assert_allclose(got["d" + key], ref, err_msg=key, **tol)


def test_gshard_rank_major_example():
    # CMU 10-423 Lecture 16 section 6.1 (b): 3 devices of capacity 3; first choices are
    # placed before second choices, so a token's second choice can find its expert full.
    idx = np.array([[0, 1], [1, 0], [1, 2], [1, 2]], np.int32)
    d = oracle.dispatch(idx, 3, 3)
    # rank 0 fills expert 1 with tokens 1, 2, 3; token 0's second choice (expert 1) is dropped
    assert d["pos"][0, 1] == 3 and d["drop"][0, 1] == 1
    assert list(d["kept"]) == [2, 3, 2]
    assert d["drop"].sum() == 1


# ---------------------------------------------------------------- experts ---

def _dense_ffn(x, w1, b1, w2, b2):
    h = np.maximum(x @ w1.T + b1, 0.0)
    return h @ w2.T + b2


def test_ffn_split_identity(golden):
    g = golden("ffn_split_identity.txt")
    n = g["n_experts"]
    rng = np.random.default_rng(11)
    d, h = 12, 10
    W = rng.standard_normal((n * h, d)).astype(np.float32)
    b = rng.standard_normal(n * h).astype(np.float32)
    U = rng.standard_normal((d, n * h)).astype(np.float32)
    c = rng.standard_normal(d).astype(np.float32)
    x = rng.standard_normal(d).astype(np.float32)
    full = oracle.expert_ffn(x, W, b, U, c)
    zeros = np.zeros(d, np.float32)
    parts_split = sum(oracle.expert_ffn(x, W[i*h:(i+1)*h], b[i*h:(i+1)*h], U[:, i*h:(i+1)*h],
                                        c if i == 0 else zeros) for i in range(n))
    parts_full_c = sum(oracle.expert_ffn(x, W[i*h:(i+1)*h], b[i*h:(i+1)*h], U[:, i*h:(i+1)*h], c)
                       for i in range(n))
    assert np.max(np.abs(parts_split - full)) < 1e-12       # the page's fp32 run: 3e-8
    np.testing.assert_allclose(parts_full_c - full, (n - 1) * c.astype(np.float64), atol=1e-12)
    # the expert is a full FFN: equals the textbook dense computation
    np.testing.assert_allclose(full, _dense_ffn(x.astype(np.float64), W.astype(np.float64),
                                                b.astype(np.float64), U.astype(np.float64),
                                                c.astype(np.float64)), rtol=1e-12, atol=1e-12)


def test_relu_expert_negative_preactivations_give_bias_only():
    d, dff = 6, 9
    x = np.ones(d, np.float32)
    w1 = -np.ones((dff, d), np.float32)
    w2 = np.random.default_rng(3).standard_normal((d, dff)).astype(np.float32)
    b2 = np.arange(d, dtype=np.float32)
    np.testing.assert_array_equal(oracle.expert_ffn(x, w1, None, w2, b2), b2.astype(np.float64))


def test_swiglu_expert_reduces_to_linear_map():
    # gate branch constant: W1 = 0, b1 = ln 3 -> silu(ln 3) = (3/4) ln 3, so the expert
    # is the linear map (3/4) ln 3 * W2 (W3 x + b3) + b2; swapping the branches fails
    rng = np.random.default_rng(4)
    d, dff = 8, 16
    x = rng.standard_normal(d).astype(np.float32)
    w1 = np.zeros((dff, d), np.float32)
    b1 = np.full(dff, np.float32(math.log(3.0)), np.float32)
    w3 = rng.standard_normal((dff, d)).astype(np.float32)
    b3 = rng.standard_normal(dff).astype(np.float32)
    w2 = rng.standard_normal((d, dff)).astype(np.float32)
    b2 = rng.standard_normal(d).astype(np.float32)
    s = float(np.float32(math.log(3.0))) / (1.0 + math.exp(-float(np.float32(math.log(3.0)))))
    want = s * (w2.astype(np.float64) @ (w3.astype(np.float64) @ x.astype(np.float64) + b3)) + b2
    got = oracle.expert_ffn(x, w1, b1, w2, b2, act=oracle.SWIGLU, w3=w3, b3=b3)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    assert abs(s - 0.75 * math.log(3.0)) < 1e-7
    # up branch constant 1 and no W3 signal: silu(W1 x + b1) through W2
    w1r = rng.standard_normal((dff, d)).astype(np.float32)
    got2 = oracle.expert_ffn(x, w1r, None, w2, None, act=oracle.SWIGLU, w3=np.zeros_like(w3),
                             b3=np.ones(dff, np.float32))
    u = w1r.astype(np.float64) @ x.astype(np.float64)
    from scipy.special import expit
    np.testing.assert_allclose(got2, w2.astype(np.float64) @ (u * expit(u)), rtol=1e-12, atol=1e-12)


def test_mixtral_expert_param_count(golden):
    g = golden("mixtral_expert_params.txt")
    d, dff = g["d_model"], g["d_ff"]
    assert round(3 * d * dff / 1e6, 1) == g["params_millions"]


# ------------------------------------------------------------ whole layer ---

def test_single_expert_layer_is_dense_ffn():
    # N = 1, C >= T: softmax over one expert is 1, nothing is dropped, and the layer
    # is the dense FFN (textbook matmuls in fp64)
    rng = np.random.default_rng(9)
    T, d, dff = 20, 16, 32
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_r = rng.standard_normal((1, d)).astype(np.float32)
    W = dict(w1=rng.standard_normal((1, dff, d)).astype(np.float32),
             b1=rng.standard_normal((1, dff)).astype(np.float32),
             w2=rng.standard_normal((1, d, dff)).astype(np.float32),
             b2=rng.standard_normal((1, d)).astype(np.float32))
    res = oracle.forward(x, w_r, None, W, k=1, C=T)
    assert np.all(res["routing"]["gate"] == 1.0)
    want = _dense_ffn(x.astype(np.float64), W["w1"][0].astype(np.float64), W["b1"][0].astype(np.float64),
                      W["w2"][0].astype(np.float64), W["b2"][0].astype(np.float64))
    np.testing.assert_allclose(res["out_exact"], want, rtol=1e-12, atol=1e-12)


def test_worked_example_layer_output(golden):
    # y = 0.366 E0(x) + 0.634 E1(x) with experts whose outputs are known in closed form:
    # W1 = I, W2 = c_i I gives E_i(x) = c_i relu(x)
    g = golden("gating_worked_example.txt")
    x = np.array([g["x"]], np.float32)
    w_r = _router_for_logits(g["x"], g["logits"])
    c = np.array([1.0, 2.0, 4.0, 8.0], np.float32)
    eye = np.eye(3, dtype=np.float32)
    W = dict(w1=np.stack([eye] * 4), w2=np.stack([ci * eye for ci in c]))
    res = oracle.forward(x, w_r, None, W, k=2, C=1)
    relu_x = np.maximum(np.array(g["x"], float), 0)
    G = np.array(g["G"], float)
    np.testing.assert_allclose(res["out_exact"][0], (G @ c.astype(float)) * relu_x, atol=2e-3)


def test_dropped_token_output_is_zero_and_rounding():
    rng = np.random.default_rng(12)
    T, d, dff, N = 30, 8, 16, 2
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_r = np.zeros((N, d), np.float32)           # everything to expert 0
    W = dict(w1=rng.standard_normal((N, dff, d)).astype(np.float32),
             w2=rng.standard_normal((N, d, dff)).astype(np.float32),
             b2=np.ones((N, d), np.float32))
    C = 7
    res = oracle.forward(x, w_r, None, W, k=1, C=C, out_dtype=oracle.BF16)
    assert np.all(res["out_exact"][C:] == 0.0)
    assert np.all(np.abs(res["out_exact"][:C]).sum(1) > 0)
    # kept tokens: gate (= 1/2 here) times the expert output, rounded once to bf16
    y = oracle.expert_ffn(x[0], W["w1"][0], None, W["w2"][0], W["b2"][0])
    np.testing.assert_allclose(res["out_exact"][0], 0.5 * y, rtol=1e-7)
    for v, rv in zip(res["out_exact"].reshape(-1), res["out"].reshape(-1)):
        assert rv == oracle.bf16_round(np.float32(v))


def test_top2_partial_drop_keeps_gate():
    # rank-0 claims fill expert 0 first; a token whose first choice overflowed keeps its
    # second assignment alone, with its original (un-renormalised) gate; a token with
    # both assignments dropped outputs zero
    T, d, dff, N = 4, 4, 8, 3
    x = np.zeros((T, d), np.float32)
    x[:, 0] = 3.0
    x[:2, 1] = 1.0
    x[2:, 2] = 2.0
    w_r = np.zeros((N, d), np.float32)
    w_r[0, 0] = 1.0
    w_r[1, 1] = 1.0
    w_r[2, 2] = 1.0
    rng = np.random.default_rng(2)
    W = dict(w1=rng.standard_normal((N, dff, d)).astype(np.float32),
             w2=rng.standard_normal((N, d, dff)).astype(np.float32))
    res = oracle.forward(x, w_r, None, W, k=2, C=1)
    r, dd = res["routing"], res["disp"]
    assert np.all(r["idx"][:, 0] == 0)
    assert list(r["idx"][:, 1]) == [1, 1, 2, 2]
    assert list(dd["drop"][:, 0]) == [0, 1, 1, 1] and list(dd["drop"][:, 1]) == [0, 1, 0, 1]
    y2 = oracle.expert_ffn(x[2], W["w1"][2], None, W["w2"][2], None)
    np.testing.assert_allclose(res["out_exact"][2], float(r["gate"][2, 1]) * y2, rtol=1e-12)
    assert r["gate"][2, 1] < 0.5
    assert np.all(res["out_exact"][3] == 0.0)
