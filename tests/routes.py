"""Independent numpy restatements of the Mamba-3 recurrence, used to pin the oracle.

Each route below is a different reading of the same statement in the Mamba-3
paper summary ("Technical Approach"); none shares code with ``oracle/``.  A
plausible oracle mistake (a dropped beta term, a rotation sign, a transposed
operand, a pair-index slip) makes at least one of them disagree.

Array layouts match the library: x [b,T,H,R,P], B/C [b,T,G,R,N], dt/A/lam
[b,T,H], theta [b,T,G,N/2], D [H], h [b,H,N,P], x_prev [b,H,R,P],
B_prev [b,G,R,N].  Everything is float64 (complex128 for the complex route).
"""
from __future__ import annotations

import numpy as np


def _heads(x, B):
    b, T, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    return b, T, H, R, P, G, N, H // G


def euler_loop(x, B, C, dt, A, D=None, h0=None):
    """Exponential-Euler (Mamba-2) recurrence, Remark 2 with lam = 1, theta = 0.

    h_t = exp(dt_t A_t) h_{t-1} + dt_t B_t x_t^T;  Y_t = h_t^T C_t + D x_t.
    """
    b, T, H, R, P, G, N, hpg = _heads(x, B)
    y = np.zeros_like(x, dtype=np.float64)
    hT = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            st = np.zeros((N, P)) if h0 is None else h0[bi, h].astype(np.float64).copy()
            Dh = 0.0 if D is None else D[h]
            for t in range(T):
                st = np.exp(dt[bi, t, h] * A[bi, t, h]) * st + \
                    dt[bi, t, h] * B[bi, t, g].T @ x[bi, t, h]
                y[bi, t, h] = (st.T @ C[bi, t, g].T).T + Dh * x[bi, t, h]
            hT[bi, h] = st
    return y, hT


def complex_route(x, B, C, dt, A, lam, theta, D=None, h0=None, x_prev=None, B_prev=None,
                  theta_is_angle=False):
    """Complex-valued SSM, "Complex-Valued State Space Models" (h in C^{N/2}).

    Transition z_t = exp(dt_t (A_t + i theta_t)); the generalised trapezoid of the
    state-input integral puts the full transition on the left endpoint:
        h_t = z_t h_{t-1} + (1 - lam_t) dt_t z_t v_{t-1} + lam_t dt_t v_t,
    with v_t = (B + i B_hat) x_t.  Readout y = Re((C + i C_hat)^T h).  The real
    projections stack as B = [B; B_hat], C = [C; -C_hat] (Proposition 2); state
    pair i is stored interleaved at (2i, 2i+1).
    """
    b, T, H, R, P, G, N, hpg = _heads(x, B)
    y = np.zeros(x.shape)
    hT = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            if h0 is None:
                hc = np.zeros((N // 2, P), dtype=np.complex128)
            else:
                hc = h0[bi, h, 0::2] + 1j * h0[bi, h, 1::2]
            if x_prev is None:
                v_prev = np.zeros((N // 2, P), dtype=np.complex128)
            else:
                bpc = B_prev[bi, g, :, 0::2] + 1j * B_prev[bi, g, :, 1::2]   # [R, N/2]
                v_prev = bpc.T @ x_prev[bi, h]                                 # [N/2, P]
            Dh = 0.0 if D is None else D[h]
            for t in range(T):
                d, a, l = dt[bi, t, h], A[bi, t, h], lam[bi, t, h]
                ang = theta[bi, t, g] if theta_is_angle else d * theta[bi, t, g]
                z = np.exp(d * a + 1j * ang)[:, None]                          # [N/2, 1]
                bc = B[bi, t, g, :, 0::2] + 1j * B[bi, t, g, :, 1::2]          # [R, N/2]
                v = bc.T @ x[bi, t, h]
                hc = z * hc + (1.0 - l) * d * z * v_prev + l * d * v
                cc = C[bi, t, g, :, 0::2] - 1j * C[bi, t, g, :, 1::2]          # C + i C_hat
                y[bi, t, h] = np.real(cc @ hc) + Dh * x[bi, t, h]
                v_prev = v
            hT[bi, h, 0::2] = hc.real
            hT[bi, h, 1::2] = hc.imag
    return y, hT


def _rot_pairs(vec, ang):
    """Rotate interleaved pairs of ``vec`` (..., N) by angles ``ang`` (N/2,)."""
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(vec)
    out[..., 0::2] = c * vec[..., 0::2] - s * vec[..., 1::2]
    out[..., 1::2] = s * vec[..., 0::2] + c * vec[..., 1::2]
    return out


def rope_route(x, B, C, dt, A, lam, theta, D=None, h0=None, x_prev=None, B_prev=None,
               theta_is_angle=False):
    """Proposition 4 read literally, in the rotated (RoPE) frame.

    psi_t = sum_{k<=t} dt_k theta_k (per pair); Q_t = R(psi_t).
        g_t = alpha_t g_{t-1} + beta_t Q_{t-1}^T B_{t-1} x_{t-1}^T + gamma_t Q_t^T B_t x_t^T
        y_t = (Q_t^T C_t)^T g_t
    with g_{-1} = h0 and Q_{-1} = I; the original-frame state is h_T = Q_T g_T.
    """
    b, T, H, R, P, G, N, hpg = _heads(x, B)
    y = np.zeros(x.shape)
    hT = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            st = np.zeros((N, P)) if h0 is None else h0[bi, h].copy()
            psi = np.zeros(N // 2)
            if x_prev is None:
                bt_prev = np.zeros((R, N))
                xprev = np.zeros((R, P))
            else:
                bt_prev = B_prev[bi, g].copy()        # rotated by Q_{-1} = I
                xprev = x_prev[bi, h]
            Dh = 0.0 if D is None else D[h]
            for t in range(T):
                d, a, l = dt[bi, t, h], A[bi, t, h], lam[bi, t, h]
                ang = theta[bi, t, g] if theta_is_angle else d * theta[bi, t, g]
                psi = psi + ang
                al = np.exp(d * a)
                be = (1.0 - l) * d * al
                ga = l * d
                bt = _rot_pairs(B[bi, t, g], -psi)    # Q_t^T B_t
                ct = _rot_pairs(C[bi, t, g], -psi)    # Q_t^T C_t
                st = al * st + be * bt_prev.T @ xprev + ga * bt.T @ x[bi, t, h]
                y[bi, t, h] = (st.T @ ct.T).T + Dh * x[bi, t, h]
                bt_prev, xprev = bt, x[bi, t, h]
            # h_T = Q_T g_T: rotate rows of the state by +psi
            hT[bi, h] = _rot_pairs(st.T, psi).T
    return y, hT


def bruteforce_txt(x, B, C, dt, A, lam, theta, D=None, theta_is_angle=False):
    """Materialised parallel form, "Parallel representation under SSD".

    Y = (L o C~ B~^T) X with L = L_decay @ L_band, where L_decay[t,s] is the
    product alpha_{s+1}..alpha_t (1 on the diagonal) and L_band holds gamma_t on
    the diagonal and beta_t on the first sub-diagonal.  B~, C~ are B, C rotated
    by the cumulative angle (Proposition 4).  Fresh sequence: h0 = 0, no
    previous token.  For MIMO the score matrix runs over (token, rank) pairs
    and L is shared by the R x R blocks.
    """
    b, T, H, R, P, G, N, hpg = _heads(x, B)
    y = np.zeros(x.shape)
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            d, a, l = dt[bi, :, h], A[bi, :, h], lam[bi, :, h]
            al = np.exp(d * a)
            be = (1.0 - l) * d * al
            ga = l * d
            Ld = np.zeros((T, T))
            for t in range(T):
                for s in range(t + 1):
                    Ld[t, s] = np.prod(al[s + 1:t + 1])
            Lb = np.diag(ga)
            for t in range(1, T):
                Lb[t, t - 1] = be[t]
            L = Ld @ Lb
            ang = theta[bi, :, g] if theta_is_angle else d[:, None] * theta[bi, :, g]
            psi = np.cumsum(ang, axis=0)                          # [T, N/2]
            bt = np.stack([_rot_pairs(B[bi, t, g], -psi[t]) for t in range(T)])  # [T,R,N]
            ct = np.stack([_rot_pairs(C[bi, t, g], -psi[t]) for t in range(T)])
            S = np.einsum("trn,usn->trus", ct, bt)                # [T,R,T,R]
            M = S * L[:, None, :, None]
            Y = np.einsum("trus,usp->trp", M, x[bi, :, h])
            Dh = 0.0 if D is None else D[h]
            y[bi, :, h] = Y + Dh * x[bi, :, h]
    return y


def bruteforce_bwd(x, B, C, dt, A, lam, theta, dy, D=None, theta_is_angle=False):
    """Reverse-mode gradients of the materialised parallel form (fresh sequence), derived by
    hand through its own quantities rather than through the recurrence:

        Y_t = sum_{s<=t} L[t,s] (C~_t . B~_s) X_s + D X_t,   C~ = R(-psi) C, B~ = R(-psi) B,
        L[t,s] = exp(cum_t - cum_s) w[t,s],  w[t,s] = gamma_s + [s < t] (1 - lam_{s+1}) dt_{s+1},
        cum_t = sum_{k<=t} dt_k A_k,  psi_t = sum_{k<=t} dt_k theta_k  ("Parallel representation
        under SSD"; Proposition 4 for the rotation).

    With G = dL/dY and S the (token, rank) score matrix: dX = (L o S)^T G + D G;
    dS = L o (G X^T); dL = <S, G X^T> per (t, s); dC~ = dS B~, dB~ = dS^T C~, rotated back by
    R(psi); dpsi_t = sum over ranks of dC~_0 C~_1 - dC~_1 C~_0 (and the same for B~), summed
    backwards over tokens into the per-step angles; dL splits into dcum (through the
    exponential) and dw (gamma_s and the next token's (1 - lam) dt), which reach dt, A and lam.
    Returns the gradients of the inputs (no starting state) as float64 arrays; B, C, theta
    gradients are summed over the heads of each group.
    """
    b, T, H, R, P, G, N, hpg = _heads(x, B)
    out = dict(dx=np.zeros(x.shape), dB=np.zeros(B.shape), dC=np.zeros(C.shape),
               ddt=np.zeros(dt.shape), dA=np.zeros(A.shape), dlam=np.zeros(lam.shape),
               dtheta=np.zeros(theta.shape), dD=None if D is None else np.zeros(D.shape))
    tri = np.tril(np.ones((T, T)))
    strict = np.tril(np.ones((T, T)), -1)
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            d, a, l = dt[bi, :, h], A[bi, :, h], lam[bi, :, h]
            cum = np.cumsum(d * a)
            E = np.exp(np.where(tri > 0, cum[:, None] - cum[None, :], 0.0)) * tri
            nxt = np.zeros(T)
            nxt[:-1] = (1.0 - l[1:]) * d[1:]
            w = (l * d)[None, :] * tri + nxt[None, :] * strict
            L = E * w
            th = theta[bi, :, g]
            ang = th if theta_is_angle else d[:, None] * th
            psi = np.cumsum(ang, axis=0)
            bt = np.stack([_rot_pairs(B[bi, t, g], -psi[t]) for t in range(T)])   # [T,R,N]
            ct = np.stack([_rot_pairs(C[bi, t, g], -psi[t]) for t in range(T)])
            S = np.einsum("trn,usn->trus", ct, bt)
            X, Gy = x[bi, :, h], dy[bi, :, h]
            Dh = 0.0 if D is None else D[h]
            M = S * L[:, None, :, None]
            out["dx"][bi, :, h] = np.einsum("trus,trp->usp", M, Gy) + Dh * Gy
            GX = np.einsum("trp,usp->trus", Gy, X)
            dS = GX * L[:, None, :, None]
            dL = np.einsum("trus,trus->tu", S, GX)
            dct = np.einsum("trus,usn->trn", dS, bt)
            dbt = np.einsum("trus,trn->usn", dS, ct)
            out["dC"][bi, :, g] += np.stack([_rot_pairs(dct[t], psi[t]) for t in range(T)])
            out["dB"][bi, :, g] += np.stack([_rot_pairs(dbt[t], psi[t]) for t in range(T)])
            dpsi = ((dct[..., 0::2] * ct[..., 1::2] - dct[..., 1::2] * ct[..., 0::2]).sum(axis=1) +
                    (dbt[..., 0::2] * bt[..., 1::2] - dbt[..., 1::2] * bt[..., 0::2]).sum(axis=1))
            dang = np.cumsum(dpsi[::-1], axis=0)[::-1]
            dE, dw = dL * w, dL * E
            dcum = (dE * E).sum(axis=1) - (dE * E).sum(axis=0)
            dga = (dw * tri).sum(axis=0)
            dnx = (dw * strict).sum(axis=0)
            ddt_, dlam_ = dga * l, dga * d
            ddt_[1:] += dnx[:-1] * (1.0 - l[1:])
            dlam_[1:] -= dnx[:-1] * d[1:]
            dda = np.cumsum(dcum[::-1])[::-1]
            ddt_ += dda * a
            if theta_is_angle:
                out["dtheta"][bi, :, g] += dang
            else:
                out["dtheta"][bi, :, g] += dang * d[:, None]
                ddt_ += (dang * th).sum(axis=1)
            out["ddt"][bi, :, h] = ddt_
            out["dA"][bi, :, h] = dda * d
            out["dlam"][bi, :, h] = dlam_
            if D is not None:
                out["dD"][h] += float((Gy * X).sum())
    return out


def chunked_bwd(x, B, C, dt, A, lam, theta, dy, chunk, D=None, h0=None, x_prev=None,
                B_prev=None, dhT=None, theta_is_angle=False):
    """Reverse-mode gradients of the chunked form, in the call's rotated frame (the algorithm
    a chunked backward runs; "Parallel representation under SSD" with Proposition 4).

    Forward, per chunk [t0, t1) with m = cum_{t0-1} (0 before the call):
        Y_t = e^{cum_t - m} C~_t^T g + sum_{s in chunk, s<=t} L[t,s] (C~_t . B~_s) X_s + D X_t
        g  <- e^{cum_{t1-1} - m} g + sum_{s in chunk} e^{cum_{t1-1} - cum_s} w_s B~_s X_s^T
    where w_s = gamma_s + (1 - lam_{s+1}) dt_{s+1} carries the next token's trapezoid share
    (w_{T-1} = gamma_{T-1}), the starting g = h0 + (1 - lam_0) dt_0 B_prev x_prev^T, and
    h_T = R(psi_{T-1}) g.  The backward keeps the adjoint of g between chunks (in reverse),
    takes the intra-chunk terms as in bruteforce_bwd, and routes every exponential, weight and
    angle to dt, A, lam and theta.  Returns all gradients, the starting state's included.
    """
    b, T, H, R, P, G, N, hpg = _heads(x, B)
    NH = N // 2
    out = dict(dx=np.zeros(x.shape), dB=np.zeros(B.shape), dC=np.zeros(C.shape),
               ddt=np.zeros(dt.shape), dA=np.zeros(A.shape), dlam=np.zeros(lam.shape),
               dtheta=np.zeros(theta.shape), dD=None if D is None else np.zeros(D.shape),
               dh0=np.zeros((b, H, N, P)), dx_prev=np.zeros((b, H, R, P)),
               dB_prev=np.zeros((b, G, R, N)))
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            d, a, l = dt[bi, :, h], A[bi, :, h], lam[bi, :, h]
            th = theta[bi, :, g]
            X, Gy = x[bi, :, h], dy[bi, :, h]
            Dh = 0.0 if D is None else D[h]
            cum = np.cumsum(d * a)
            ang = th if theta_is_angle else d[:, None] * th
            psi = np.cumsum(ang, axis=0)
            bt = np.stack([_rot_pairs(B[bi, t, g], -psi[t]) for t in range(T)])   # [T,R,N]
            ct = np.stack([_rot_pairs(C[bi, t, g], -psi[t]) for t in range(T)])
            w = l * d
            w[:-1] = w[:-1] + (1.0 - l[1:]) * d[1:]
            xp0 = np.zeros((R, P)) if x_prev is None else x_prev[bi, h]
            bp0 = np.zeros((R, N)) if B_prev is None else B_prev[bi, g]
            g0 = (np.zeros((N, P)) if h0 is None else h0[bi, h].copy())
            g0 = g0 + (1.0 - l[0]) * d[0] * np.einsum("rn,rp->np", bp0, xp0)
            bounds = list(range(0, T, chunk)) + [T]
            chunks = list(zip(bounds[:-1], bounds[1:]))
            # forward: the state entering every chunk
            gin, gs = [], g0
            for t0, t1 in chunks:
                gin.append(gs)
                m = cum[t0 - 1] if t0 > 0 else 0.0
                V = np.einsum("s,srn,srp->np", np.exp(cum[t1 - 1] - cum[t0:t1]) * w[t0:t1],
                              bt[t0:t1], X[t0:t1])
                gs = np.exp(cum[t1 - 1] - m) * gs + V
            gT = gs
            hT = _rot_pairs(gT.T, psi[T - 1]).T                              # [N,P]
            # reverse
            dX, dbt, dct = Dh * Gy, np.zeros(bt.shape), np.zeros(ct.shape)
            dcum, dw, dpsi = np.zeros(T), np.zeros(T), np.zeros((T, NH))
            dga_i, dnx_i = np.zeros(T), np.zeros(T)        # intra-chunk band weights
            if dhT is not None:
                dH = dhT[bi, h]
                dg = _rot_pairs(dH.T, -psi[T - 1]).T
                dpsi[T - 1] += (dH[1::2] * hT[0::2] - dH[0::2] * hT[1::2]).sum(axis=1)
            else:
                dg = np.zeros((N, P))
            for (t0, t1), gi in zip(chunks[::-1], gin[::-1]):
                m = cum[t0 - 1] if t0 > 0 else 0.0
                # state update
                Eend = np.exp(cum[t1 - 1] - m)
                dgin = Eend * dg
                q = Eend * float((dg * gi).sum())
                dcum[t1 - 1] += q
                if t0 > 0:
                    dcum[t0 - 1] -= q
                for s in range(t0, t1):
                    es = np.exp(cum[t1 - 1] - cum[s])
                    Vs = np.einsum("rn,rp->np", bt[s], X[s])
                    dv = float((dg * Vs).sum())
                    dw[s] += es * dv
                    dcum[t1 - 1] += es * w[s] * dv
                    dcum[s] -= es * w[s] * dv
                    dbt[s] += es * w[s] * np.einsum("np,rp->rn", dg, X[s])
                    dX[s] += es * w[s] * np.einsum("rn,np->rp", bt[s], dg)
                # inter-chunk output: e^{cum_t - m} C~_t^T g_in
                for t in range(t0, t1):
                    f = np.exp(cum[t] - m)
                    Z = np.einsum("rn,np->rp", ct[t], gi)
                    dct[t] += f * np.einsum("np,rp->rn", gi, Gy[t])
                    dgin += f * np.einsum("rn,rp->np", ct[t], Gy[t])
                    q = f * float((Gy[t] * Z).sum())
                    dcum[t] += q
                    if t0 > 0:
                        dcum[t0 - 1] -= q
                # intra-chunk: L[t,s] = e^{cum_t - cum_s}(gamma_s + [s<t](1 - lam_{s+1}) dt_{s+1})
                n = t1 - t0
                tri = np.tril(np.ones((n, n)))
                strict = np.tril(np.ones((n, n)), -1)
                cc = cum[t0:t1]
                E = np.exp(np.where(tri > 0, cc[:, None] - cc[None, :], 0.0)) * tri
                nx = np.zeros(n)
                nx[:-1] = (1.0 - l[t0 + 1:t1]) * d[t0 + 1:t1]
                om = (l[t0:t1] * d[t0:t1])[None, :] * tri + nx[None, :] * strict
                L = E * om
                S = np.einsum("trn,usn->trus", ct[t0:t1], bt[t0:t1])
                GX = np.einsum("trp,usp->trus", Gy[t0:t1], X[t0:t1])
                dX[t0:t1] += np.einsum("trus,trp->usp", S * L[:, None, :, None], Gy[t0:t1])
                dS = GX * L[:, None, :, None]
                dL = np.einsum("trus,trus->tu", S, GX)
                dct[t0:t1] += np.einsum("trus,usn->trn", dS, bt[t0:t1])
                dbt[t0:t1] += np.einsum("trus,trn->usn", dS, ct[t0:t1])
                dE, dom = dL * om, dL * E
                dcum[t0:t1] += (dE * E).sum(axis=1) - (dE * E).sum(axis=0)
                dga_i[t0:t1] += (dom * tri).sum(axis=0)
                dnx_i[t0:t1] += (dom * strict).sum(axis=0)
                dg = dgin
            # the starting state g0 = h0 + (1 - lam_0) dt_0 B_prev x_prev^T
            out["dh0"][bi, h] = dg
            k0 = (1.0 - l[0]) * d[0]
            v0 = float((dg * np.einsum("rn,rp->np", bp0, xp0)).sum())
            out["dx_prev"][bi, h] = k0 * np.einsum("rn,np->rp", bp0, dg)
            out["dB_prev"][bi, g] += k0 * np.einsum("np,rp->rn", dg, xp0)
            # rotation back, angles
            out["dC"][bi, :, g] += np.stack([_rot_pairs(dct[t], psi[t]) for t in range(T)])
            out["dB"][bi, :, g] += np.stack([_rot_pairs(dbt[t], psi[t]) for t in range(T)])
            dpsi += ((dct[..., 0::2] * ct[..., 1::2] - dct[..., 1::2] * ct[..., 0::2]).sum(axis=1) +
                     (dbt[..., 0::2] * bt[..., 1::2] - dbt[..., 1::2] * bt[..., 0::2]).sum(axis=1))
            dang = np.cumsum(dpsi[::-1], axis=0)[::-1]
            # coefficients: w (state), the intra band weights, gamma, cum
            ddt_, dlam_ = np.zeros(T), np.zeros(T)
            dga = dw + dga_i
            dnx = dnx_i.copy()
            dnx[:-1] += dw[:-1]
            ddt_ += dga * l
            dlam_ += dga * d
            ddt_[1:] += dnx[:-1] * (1.0 - l[1:])
            dlam_[1:] -= dnx[:-1] * d[1:]
            ddt_[0] += (1.0 - l[0]) * v0
            dlam_[0] -= d[0] * v0
            dda = np.cumsum(dcum[::-1])[::-1]
            ddt_ += dda * a
            if theta_is_angle:
                out["dtheta"][bi, :, g] += dang
            else:
                out["dtheta"][bi, :, g] += dang * d[:, None]
                ddt_ += (dang * th).sum(axis=1)
            out["dx"][bi, :, h] = dX
            out["ddt"][bi, :, h] = ddt_
            out["dA"][bi, :, h] = dda * d
            out["dlam"][bi, :, h] = dlam_
            if D is not None:
                out["dD"][h] += float((Gy * X).sum())
    return out


def implicit_conv_route(x, B, C, dt, A, lam, D=None, h0=None, x_prev=None, B_prev=None):
    """Remark 4 (theta = 0): width-2 data-dependent convolution on v_t = B_t x_t^T,

        v~_t = beta_t v_{t-1} + gamma_t v_t,   h_t = alpha_t h_{t-1} + v~_t.
    """
    b, T, H, R, P, G, N, hpg = _heads(x, B)
    y = np.zeros(x.shape)
    hT = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            st = np.zeros((N, P)) if h0 is None else h0[bi, h].copy()
            v_prev = np.zeros((N, P)) if x_prev is None else B_prev[bi, g].T @ x_prev[bi, h]
            Dh = 0.0 if D is None else D[h]
            for t in range(T):
                d, a, l = dt[bi, t, h], A[bi, t, h], lam[bi, t, h]
                al = np.exp(d * a)
                v = B[bi, t, g].T @ x[bi, t, h]
                vt = (1.0 - l) * d * al * v_prev + l * d * v
                st = al * st + vt
                y[bi, t, h] = (st.T @ C[bi, t, g].T).T + Dh * x[bi, t, h]
                v_prev = v
            hT[bi, h] = st
    return y, hT


def lti_exact(a, b, omega, tau):
    """Exact solution of h' = a h + b sin(omega tau), h(0) = 0 (variation of constants)."""
    return b * (omega * np.exp(a * tau) - omega * np.cos(omega * tau) - a * np.sin(omega * tau)) \
        / (a * a + omega * omega)
