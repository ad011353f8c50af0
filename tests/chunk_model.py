"""fp64 numpy model of the chunkwise-parallel form the CUDA prefill kernel computes.

Tests only: it is NOT the oracle.  It exists to check, on the CPU and before any
kernel runs, that the chunk algebra the kernel is built on reproduces the token
recurrence, including the worst-case decay g = -5 everywhere, and to predict the
size of the error that bf16 operands introduce (`bf16=True` rounds every tensor-core
operand to bf16 at the same points the kernel does).

Per head, chunk of C tokens, local index r, state S (dk x dv) at the chunk start:

  Gam_r = sum_{t <= r} g_t (per channel);  Kt_r = k_r * exp(Gam_r);  Qt_r = q_r * exp(Gam_r)
  Kb_j  = k_j * exp(Gam_C - Gam_j)
  A_rj  = beta_r * sum_i k_r[i] k_j[i] exp(Gam_r[i] - Gam_j[i])          (j < r)
  P_rj  =          sum_i q_r[i] k_j[i] exp(Gam_r[i] - Gam_j[i])          (j <= r)
  U     = (I + A)^-1 Diag(beta) (V - Kt S)
  O     = Qt S + P U
  S'    = Diag(exp Gam_C) S + Kb^T U

The products exp(Gam_r - Gam_j) are never formed from exp(Gam_r) * exp(-Gam_j) over a
whole chunk (that overflows for C = 64 at g = -5).  The kernel splits the chunk into
sub-blocks of `sub` tokens.  For a pair of distinct sub-blocks (R > J) it factors the decay
at the last token of block J, so both factors are <= 1.  Within a diagonal block it factors
at the block's middle token, so each factor is at most exp(5 * sub / 2), which is below
the fp32/bf16 range for sub <= 32 because the log-decay is bounded below by -5 (the
bound the skill card's quick facts attribute to the scaled-sigmoid gate, which is what
lets the diagonal tiles run as dense tensor-core products).
"""
import numpy as np


def _bf16(x):
    """Round fp64 -> bf16 (round to nearest even via fp32), back to fp64."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    out = u.astype(np.uint32).view(np.float32).astype(np.float64)
    # keep inf/nan as they are
    bad = ~np.isfinite(f)
    out[bad] = f[bad]
    return out


def _ftz(x):
    """Flush magnitudes below the smallest normal fp32 number to zero (as the kernel's ex2 does)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(np.abs(x) < 2.0 ** -126, 0.0, x)


def kernel_inverse(A, rnd):
    """(I + A)^-1 for a strictly lower 64x64 A the way the tensor-core kernel forms it.

    Diagonal 16x16 blocks: N = A_bb is nilpotent, (I + N)^-1 = (I - N)(I + N^2)(I + N^4)(I + N^8),
    every product with operands rounded by `rnd` and exact sums.  Off-diagonal blocks: At_RL =
    X_RR A_RL, then X_RJ = -sum_{L=J}^{R-1} At_RL X_LJ down each block column, operands rounded.
    """
    n = A.shape[0]
    nb = n // 16
    X = np.zeros_like(A)
    I16 = np.eye(16)
    for b in range(nb):
        s = slice(16 * b, 16 * b + 16)
        N = A[s, s]
        P = I16 - N
        Np = N
        for _ in range(3):
            Np = rnd(Np) @ rnd(Np)
            P = P + rnd(P) @ rnd(Np)
        X[s, s] = P
    # off-diagonal blocks: At_RL = X_RR A_RL first (operands rounded, result rounded as the next
    # product's operand), then X_RJ = -sum_{L=J}^{R-1} At_RL X_LJ down each block column
    At = {}
    for R in range(nb):
        for L in range(R):
            At[(R, L)] = rnd(rnd(X[16 * R:16 * R + 16, 16 * R:16 * R + 16]) @ rnd(A[16 * R:16 * R + 16, 16 * L:16 * L + 16]))
    for J in range(nb):
        js = slice(16 * J, 16 * J + 16)
        for R in range(J + 1, nb):
            X[16 * R:16 * R + 16, js] = -sum(At[(R, L)] @ rnd(X[16 * L:16 * L + 16, js]) for L in range(J, R))
    return X


def chunk_head(q, k, v, g, beta, S0, C=64, sub=32, bf16=False, offdiag_ref="block_end", solve="exact"):
    """One head. q,k,g [T,dk]; v [T,dv]; beta [T]; S0 [dk,dv]. Returns (o [T,dv], S_T).

    offdiag_ref: reference token of an off-diagonal block pair (R > J).  "block_end" factors at
    the last token of block J (both factors <= 1: exact).  "row_middle" factors at the middle
    token of block R, the same reference as the diagonal block of R, and flushes column factors
    below the fp32 normal range to zero: this is what the tensor-core kernel does for C = 64,
    sub = 32 (one product for the whole block row).  The kernel builds those column factors from
    in-range pieces, so it flushes no more than this model does.

    solve: "exact" solves (I + A) T = Diag(beta) in fp64; "kernel" forms (I + A)^-1 as the tensor-core
    kernel does (kernel_inverse, with the bf16 rounding when bf16=True; needs C = 64).
    """
    T, dk = q.shape
    dv = v.shape[1]
    rnd = _bf16 if bf16 else (lambda x: x)
    S = np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    assert C % sub == 0
    for c0 in range(0, T, C):
        n = min(C, T - c0)
        qc = np.zeros((C, dk)); kc = np.zeros((C, dk)); gc = np.zeros((C, dk))
        vc = np.zeros((C, dv)); bc = np.zeros(C)
        qc[:n], kc[:n], gc[:n], vc[:n], bc[:n] = q[c0:c0 + n], k[c0:c0 + n], g[c0:c0 + n], v[c0:c0 + n], beta[c0:c0 + n]
        Gam = np.cumsum(gc, axis=0)
        A = np.zeros((C, C))
        P = np.zeros((C, C))
        nb = C // sub
        for R in range(nb):
            rows = slice(R * sub, (R + 1) * sub)
            for J in range(R + 1):
                cols = slice(J * sub, (J + 1) * sub)
                if J == R or offdiag_ref == "row_middle":
                    ref = Gam[R * sub + sub // 2]
                else:
                    ref = Gam[J * sub + sub - 1]
                with np.errstate(over="ignore"):
                    er = np.exp(Gam[rows] - ref)
                    ej = np.exp(ref - Gam[cols])
                if J != R and offdiag_ref == "row_middle":
                    ej = _ftz(ej)
                # the kernel multiplies the bf16 q and k by bf16-rounded factors (two roundings), except
                # the block-1 x block-0 columns, which it forms in fp32 (one rounding)
                qs = rnd(qc[rows] * rnd(er))
                ks = rnd(kc[rows] * rnd(er))
                kh = rnd(kc[cols] * ej) if J != R else rnd(kc[cols] * rnd(ej))
                P[rows, cols] = qs @ kh.T
                A[rows, cols] = ks @ kh.T
        with np.errstate(invalid="ignore", over="ignore"):
            P = np.where(np.tril(np.ones((C, C), bool)), P, 0.0)
            A = np.where(np.tril(np.ones((C, C), bool), -1), A, 0.0) * bc[:, None]
        if solve == "kernel":
            Tm = kernel_inverse(A, rnd) * bc[None, :]
        else:
            Tm = np.linalg.solve(np.eye(C) + A, np.diag(bc))
        if bf16:
            # the kernel forms these as the bf16 tile against the block's reference token times
            # bf16 e^{Gam_ref}: two roundings
            refs = np.repeat(Gam[sub // 2::sub], sub, axis=0)
            with np.errstate(over="ignore"):
                Kt = rnd(rnd(kc * rnd(np.exp(Gam - refs))) * rnd(np.exp(refs)))
                Qt = rnd(rnd(qc * rnd(np.exp(Gam - refs))) * rnd(np.exp(refs)))
        else:
            Kt = kc * np.exp(Gam)
            Qt = qc * np.exp(Gam)
        Kb = rnd(kc * np.exp(Gam[-1] - Gam))
        Sb = rnd(S)
        Y = vc - Kt @ Sb
        U = rnd(Tm) @ rnd(Y)
        Ub = rnd(U)
        O = Qt @ Sb + rnd(P) @ Ub
        S = np.exp(Gam[-1])[:, None] * S + Kb.T @ Ub
        o[c0:c0 + n] = O[:n]
    return o, S


def chunk_forward(q, k, v, g, beta, S0=None, C=64, sub=32, bf16=False, offdiag_ref="block_end", solve="exact"):
    """[B,T,H,*] fp64 arrays -> (o [B,T,H,dv], S_T [B,H,dk,dv])."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            s0 = np.zeros((dk, dv)) if S0 is None else S0[b, h]
            o[b, :, h], ST[b, h] = chunk_head(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h],
                                              beta[b, :, h], s0, C=C, sub=sub, bf16=bf16,
                                              offdiag_ref=offdiag_ref, solve=solve)
    return o, ST
