"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics, not by the oracle.

Each pin takes the oracle's (forward, decode_step) pair and raises AssertionError when the
oracle disagrees.  The same functions run against deliberately broken copies of the
oracle in test_oracle_mutants.py, to show that a plausible mistake fails at least one pin.

Pins (numbering as in the design notes):
  I1  beta = 0, S0 = 0  ->  o == 0 and S_T == 0 exactly.
  I2  beta = 0, S0 != 0 ->  pure decay: o_t = S0^T (exp(Gam_t) * q_t), S_T = Diag(exp Gam_T) S0.
  I3  one token, S0 = 0 ->  o_1 = beta (q.k) v.
  I4  g = 0, beta = 1, orthonormal keys, S0 = 0 -> querying with k_i returns v_i.
  I5  g = 0, beta = 1, the same unit key written twice -> the second value overwrites the first.
  I6  tokens with beta = 0 and g = 0 leave the state unchanged (padding is a no-op).
  I7  splitting the sequence and carrying the state gives the same result.
  I8  T single-token decode steps equal one forward over the same T tokens.
  I9  (o, S_T) is linear in (S0, V) for fixed q, k, g, beta.
  I10 with unit keys and beta in (0,1): ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t||.
  I11 agreement with an independent dense-matrix-product unrolling on tiny inputs.
  G1  the hand-worked three-token example in tests/golden/hand_worked_dk2.json.
"""
import json
import os

import numpy as np

from helpers import max_rel_err, random_problem, unit_rows

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pin_I1_beta_zero(fwd, dec, rng):
    q, k, v, g, beta, _ = random_problem(rng, 2, 37, 3, 8, 6, s0=False)
    o, ST = fwd(q, k, v, g, np.zeros_like(beta), None)
    assert np.all(o == 0.0) and np.all(ST == 0.0), "beta=0 with S0=0 must give exactly zero"


def pin_I2_pure_decay(fwd, dec, rng):
    q, k, v, g, beta, S0 = random_problem(rng, 1, 23, 2, 7, 5)
    o, ST = fwd(q, k, v, g, np.zeros_like(beta), S0)
    Gam = np.cumsum(g, axis=1)                                   # [B,T,H,dk]
    o_ref = np.einsum("bhic,bthi->bthc", S0, np.exp(Gam) * q)
    ST_ref = np.exp(Gam[:, -1])[..., None] * S0                  # [B,H,dk,1] * [B,H,dk,dv]
    assert max_rel_err(o, o_ref) < 1e-12, max_rel_err(o, o_ref)
    assert max_rel_err(ST, ST_ref) < 1e-12, max_rel_err(ST, ST_ref)


def pin_I3_single_token(fwd, dec, rng):
    q, k, v, g, beta, _ = random_problem(rng, 3, 1, 4, 16, 12, s0=False)
    o, ST = fwd(q, k, v, g, beta, None)
    qk = np.einsum("bthi,bthi->bth", q, k)
    o_ref = (beta * qk)[..., None] * v
    ST_ref = np.einsum("bhi,bhc->bhic", k[:, 0], (beta[..., None] * v)[:, 0])
    assert max_rel_err(o, o_ref) < 1e-13, max_rel_err(o, o_ref)
    assert max_rel_err(ST, ST_ref) < 1e-13, max_rel_err(ST, ST_ref)


def pin_I4_orthonormal_recall(fwd, dec, rng):
    dk, dv, n = 12, 9, 10
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :n].T                                           # n orthonormal rows
    vals = rng.standard_normal((n, dv))
    T = 2 * n
    q = np.zeros((1, T, 1, dk)); k = np.zeros((1, T, 1, dk)); v = np.zeros((1, T, 1, dv))
    g = np.zeros((1, T, 1, dk)); beta = np.zeros((1, T, 1))
    perm = rng.permutation(n)
    for t in range(n):                                           # write phase
        k[0, t, 0] = keys[t]; v[0, t, 0] = vals[t]; beta[0, t, 0] = 1.0
        q[0, t, 0] = unit_rows(rng, (dk,))
    for t in range(n):                                           # read phase (beta = 0: no write)
        q[0, n + t, 0] = keys[perm[t]]
        k[0, n + t, 0] = unit_rows(rng, (dk,))
    o, _ = fwd(q, k, v, g, beta, None)
    got = o[0, n:, 0]
    assert np.max(np.abs(got - vals[perm])) < 1e-12, np.max(np.abs(got - vals[perm]))


def pin_I5_overwrite(fwd, dec, rng):
    dk, dv = 6, 4
    key = unit_rows(rng, (dk,))
    v1, v2 = rng.standard_normal(dv), rng.standard_normal(dv)
    q = unit_rows(rng, (1, 2, 1, dk))
    k = np.stack([key, key])[None, :, None]
    v = np.stack([v1, v2])[None, :, None]
    g = np.zeros((1, 2, 1, dk)); beta = np.ones((1, 2, 1))
    _, ST = fwd(q, k, v, g, beta, None)
    assert max_rel_err(ST[0, 0], np.outer(key, v2)) < 1e-13


def pin_I6_padding(fwd, dec, rng):
    q, k, v, g, beta, S0 = random_problem(rng, 1, 20, 2, 8, 8)
    o, ST = fwd(q, k, v, g, beta, S0)
    ins = [0, 5, 6, 13, 20]                                      # insert no-op tokens before these
    keep = []
    qs, ks, vs, gs, bs = [], [], [], [], []
    t = 0
    for pos in range(21):
        if pos in ins:
            qs.append(unit_rows(rng, (1, 1, 2, 8))); ks.append(unit_rows(rng, (1, 1, 2, 8)))
            vs.append(rng.standard_normal((1, 1, 2, 8))); gs.append(np.zeros((1, 1, 2, 8)))
            bs.append(np.zeros((1, 1, 2))); t += 1
        if pos < 20:
            qs.append(q[:, pos:pos + 1]); ks.append(k[:, pos:pos + 1]); vs.append(v[:, pos:pos + 1])
            gs.append(g[:, pos:pos + 1]); bs.append(beta[:, pos:pos + 1]); keep.append(t); t += 1
    o2, ST2 = fwd(*(np.concatenate(x, axis=1) for x in (qs, ks, vs, gs, bs)), S0)
    assert max_rel_err(ST2, ST) < 1e-13
    assert max_rel_err(o2[:, keep], o) < 1e-13


def pin_I7_split_resume(fwd, dec, rng):
    q, k, v, g, beta, S0 = random_problem(rng, 2, 50, 2, 8, 5)
    o, ST = fwd(q, k, v, g, beta, S0)
    for T1 in (1, 17, 49):
        oa, Sa = fwd(q[:, :T1], k[:, :T1], v[:, :T1], g[:, :T1], beta[:, :T1], S0)
        ob, Sb = fwd(q[:, T1:], k[:, T1:], v[:, T1:], g[:, T1:], beta[:, T1:], Sa)
        assert max_rel_err(np.concatenate([oa, ob], axis=1), o) < 1e-13
        assert max_rel_err(Sb, ST) < 1e-13


def pin_I8_decode_equals_forward(fwd, dec, rng):
    q, k, v, g, beta, S0 = random_problem(rng, 3, 9, 2, 8, 4)
    o, ST = fwd(q, k, v, g, beta, S0)
    S = np.array(S0)
    for t in range(9):
        ot = dec(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S)
        assert max_rel_err(ot, o[:, t]) < 1e-13
    assert max_rel_err(S, ST) < 1e-13


def pin_I9_linearity(fwd, dec, rng):
    q, k, v, g, beta, S0 = random_problem(rng, 1, 30, 2, 8, 8)
    o1, S1 = fwd(q, k, v, g, beta, S0)
    o2, S2 = fwd(q, k, 2.5 * v, g, beta, 2.5 * S0)
    assert max_rel_err(o2, 2.5 * o1) < 1e-13 and max_rel_err(S2, 2.5 * S1) < 1e-13
    # additivity: (V, S0) = (V_a + V_b, S0_a + S0_b)
    vb = rng.standard_normal(v.shape); Sb0 = rng.standard_normal(S0.shape)
    oa, Sa = fwd(q, k, v, g, beta, S0)
    ob, Sb = fwd(q, k, vb, g, beta, Sb0)
    oc, Sc = fwd(q, k, v + vb, g, beta, S0 + Sb0)
    assert max_rel_err(oc, oa + ob) < 1e-12 and max_rel_err(Sc, Sa + Sb) < 1e-12


def pin_I10_boundedness(fwd, dec, rng):
    q, k, v, g, beta, S0 = random_problem(rng, 1, 40, 1, 8, 8)
    S = np.array(S0)
    for t in range(40):
        before = np.linalg.norm(S[0, 0])
        dec(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S)
        after = np.linalg.norm(S[0, 0])
        assert after <= before + beta[0, t, 0] * np.linalg.norm(v[0, t, 0]) + 1e-12


def dense_unrolling(q, k, v, g, beta, S0):
    """Independent formulation: explicit transition matrices and their products.

    M_t = (I - beta_t k_t k_t^T) Diag(exp g_t);  S_t = Phi_{t,0} S0 + sum_{j<=t} Phi_{t,j} beta_j k_j v_j^T,
    with Phi_{t,j} = M_t ... M_{j+1} (Phi_{t,t} = I);  o_t = S_t^T q_t.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            Ms = [(np.eye(dk) - beta[b, t, h] * np.outer(k[b, t, h], k[b, t, h])) @ np.diag(np.exp(g[b, t, h]))
                  for t in range(T)]
            for t in range(T):
                def phi(j):  # M_t ... M_{j+1}, as a product of matrices, newest on the left
                    P = np.eye(dk)
                    for s in range(j + 1, t + 1):
                        P = Ms[s] @ P
                    return P
                St = phi(-1) @ S0[b, h]
                for j in range(t + 1):
                    St = St + phi(j) @ np.outer(beta[b, j, h] * k[b, j, h], v[b, j, h])
                o[b, t, h] = St.T @ q[b, t, h]
                if t == T - 1:
                    ST[b, h] = St
    return o, ST


def pin_I11_dense_unrolling(fwd, dec, rng):
    for (T, dk, dv) in ((1, 3, 2), (5, 4, 3), (8, 8, 5)):
        q, k, v, g, beta, S0 = random_problem(rng, 2, T, 2, dk, dv)
        o, ST = fwd(q, k, v, g, beta, S0)
        o_ref, ST_ref = dense_unrolling(q, k, v, g, beta, S0)
        assert max_rel_err(o, o_ref) < 1e-12, max_rel_err(o, o_ref)
        assert max_rel_err(ST, ST_ref) < 1e-12, max_rel_err(ST, ST_ref)


def pin_G1_hand_worked(fwd, dec, rng):
    with open(os.path.join(GOLDEN, "hand_worked_dk2.json")) as f:
        gold = json.load(f)
    def lift(x):
        return np.asarray(x, dtype=np.float64)[None, :, None]
    q, k, v = lift(gold["q"]), lift(gold["k"]), lift(gold["v"])
    g = np.log(lift(gold["exp_g"]))
    beta = np.asarray(gold["beta"], dtype=np.float64)[None, :, None]
    o, ST = fwd(q, k, v, g, beta, None)
    assert np.max(np.abs(o[0, :, 0] - np.asarray(gold["o"]))) < 1e-12
    assert np.max(np.abs(ST[0, 0] - np.asarray(gold["S_T"]))) < 1e-12


ALL_PINS = [pin_I1_beta_zero, pin_I2_pure_decay, pin_I3_single_token, pin_I4_orthonormal_recall,
            pin_I5_overwrite, pin_I6_padding, pin_I7_split_resume, pin_I8_decode_equals_forward,
            pin_I9_linearity, pin_I10_boundedness, pin_I11_dense_unrolling, pin_G1_hand_worked]
