"""Pins for the fp64 KDA oracle: checks against what the recurrence fixes
independently of the oracle's own code.

Each ``pin_*`` takes an oracle library handle (so the planted-mutation test
can run the same battery against deliberately broken builds of the oracle)
and raises AssertionError on failure.  Inputs are small and seeded.

What pins what (recurrence: delta rule with a channel-wise forget gate, CSDN
post on the Kimi K3 technical report, section 一.1):
  * pin_identity_beta0        beta=0, alpha=1 leaves the state unchanged, o = S0^T q
  * pin_orthonormal_retrieval beta=1, alpha=1, orthonormal keys: S^T k_j = v_j exactly
  * pin_self_query            beta=1, |k|=1, q=k gives o_t = v_t for any S and alpha
  * pin_decay_closed_form     beta=0: S_t = Diag(exp(G_t)) S_0 (closed form)
  * pin_golden_fixtures       hand-worked values under tests/golden/
  * pin_brute_force           dense (I - beta k k^T) Diag(alpha) products, tiny T and d
  * pin_chunked_form          chunk-parallel algebra ("Kimi K3 开源日来了", FlashKDA
                              section: parallel inside a chunk, serial between chunks)
                              equals the oracle for C in {1, 16, 64, T}
  * pin_split_combine         zero-start state + transition, combined, equals the
                              unsplit run ("Kimi K3 开源日来了", Infra section, first layer)
  * pin_snapshot_tagging      snapshots hold exactly the first j*stride tokens
  * pin_contraction_bound     ||S_t|| <= ||S_{t-1}|| + beta ||k|| ||v||
  * pin_resume                prefill(0..L) == prefill(jS..L) started from snapshot j
  * pin_decode_matches_prefill L decode steps == a prefill of L tokens
  * pin_decode_slots          decode writes the slot it is told to and no other
  * pin_varlen_isolation      a packed request equals the same request run alone
  * pin_gate_logit_map        the fused gate activation log(alpha) = -5 sigmoid(x):
                              exact values, the reflection g(x) + g(-x) = -5, the
                              range, and its slope against central differences
  * pin_gate_logit_decay      beta = 0 with zero logits: S_t = exp(-2.5 t) S_0
  * pin_gate_logit_backward   the logits' gradient against central differences of
                              the forward loss in the logits
"""
from __future__ import annotations

import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_inputs(lengths, H, dk, dv, seed=0, gate_lo=-5.0, s0_std=None):
    rng = _rng(seed)
    T = int(sum(lengths))
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    g = gate_lo * (1.0 / (1.0 + np.exp(-rng.standard_normal((T, H, dk)))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    s0 = None if s0_std is None else s0_std * rng.standard_normal((len(lengths), H, dk, dv))
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu=cu, s0=s0)


def _run(lib, x, stride=0, n_threads=2):
    return oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu"], x["s0"],
                          snapshot_stride=stride, n_threads=n_threads, lib=lib)


# ----------------------------------------------------------------------------
# Independent restatements used as pins (written from the definition, not from
# the oracle source).
# ----------------------------------------------------------------------------

def brute_force_chain(q, k, v, g, beta, s0):
    """Dense transition matrices: S_t = A_t S_{t-1} + beta k v^T with
    A_t = (I - beta_t k_t k_t^T) Diag(alpha_t).  Returns (o [L,dv], states [L,dk,dv])."""
    L, dk = k.shape
    S = s0.copy()
    outs, states = [], []
    for t in range(L):
        A = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t]))
        S = A @ S + beta[t] * np.outer(k[t], v[t])
        outs.append(S.T @ q[t])
        states.append(S.copy())
    return np.array(outs), np.array(states)


def chunked_chain(q, k, v, g, beta, s0, C):
    """Chunk-parallel form derived by unrolling the recurrence inside a chunk.

    With G_t = sum_{s<=t} g_s (chunk-local) and gamma_t = exp(G_t):
      A_ij = sum_c k_ic k_jc exp(G_ic - G_jc)  (j < i),  P_ij = same with q_i (j <= i)
      (I + Diag(beta) A) U = Diag(beta) (V - (gamma*K) S0)
      O = (gamma*Q) S0 + P U,   S_C = Diag(gamma_C) S0 + ((gamma_C/gamma)*K)^T U
    The exponent differences are formed before exponentiation, so nothing
    over- or underflows in fp64 at these sizes.
    """
    L, dk = k.shape
    dv = v.shape[1]
    S = s0.copy()
    O = np.zeros((L, dv))
    for c0 in range(0, L, C):
        sl = slice(c0, min(c0 + C, L))
        K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
        n = K.shape[0]
        G = np.cumsum(g[sl], axis=0)
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        D = G[:, None, :] - G[None, :, :]
        D = np.where((ii >= jj)[:, :, None], D, -np.inf)
        E = np.exp(D)
        A = np.einsum("ic,jc,ijc->ij", K, K, E) * (ii > jj)
        P = np.einsum("ic,jc,ijc->ij", Q, K, E) * (ii >= jj)
        gam = np.exp(G)
        Tinv = np.linalg.inv(np.eye(n) + b[:, None] * A)
        W = Tinv @ (b[:, None] * gam * K)
        Ut = Tinv @ (b[:, None] * V)
        U = Ut - W @ S
        O[sl] = (gam * Q) @ S + P @ U
        tail = np.exp(G[-1][None, :] - G)
        S = np.exp(G[-1])[:, None] * S + (tail * K).T @ U
    return O, S


def chunked_backward_chain(q, k, v, g, beta, s0, d_o, d_fin, C):
    """The backward of chunked_chain, derived by reverse mode through its
    chunk algebra (one chain).  Returns dict(dq, dk, dv, dg, dbeta, d_initial).

    Per chunk, with S its start state, dSn the cotangent of its end state,
    Gam = gamma at the chunk's last token and Khat = (Gam / gamma) * K:
      dU  = P^T dO + Khat dSn
      dS  = Diag(Gam) dSn + (gamma Q)^T dO - W^T dU            (serial, chunks in reverse)
      dP  = tril(dO U^T),  d(gamma Q) = dO S^T,  dKhat = U dSn^T,  dW = -dU S^T
      [U~ | W] = T Diag(beta) [V | gamma K]  ->  dV, d(gamma K), dT, dbeta
      T = (I + Diag(beta) A)^-1  ->  dZ = -T^T dT T^T,  dA = tril_strict(Diag(beta) dZ)
      A, P gated products -> dK, dQ and the cumulative-gate cotangent dG, every
      gate factor an exp(G_t - G_s) with t >= s (never above 1);
      dg = reverse cumulative sum of dG inside the chunk.
    """
    L, dk = k.shape
    dv = v.shape[1]
    starts = list(range(0, L, C))
    # forward: chunk-start states and the chunk quantities the backward reuses
    S = s0.copy()
    fw = []
    for c0 in starts:
        sl = slice(c0, min(c0 + C, L))
        K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
        n = K.shape[0]
        G = np.cumsum(g[sl], axis=0)
        ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        D = np.where((ii >= jj)[:, :, None], G[:, None, :] - G[None, :, :], -np.inf)
        E = np.exp(D)                                   # E[t, s, c] = exp(G_tc - G_sc), t >= s
        A = np.einsum("ic,jc,ijc->ij", K, K, E) * (ii > jj)
        P = np.einsum("ic,jc,ijc->ij", Q, K, E) * (ii >= jj)
        gam = np.exp(G)
        Gam = gam[-1]
        T = np.linalg.inv(np.eye(n) + b[:, None] * A)
        Kg, Qg = gam * K, gam * Q
        W = T @ (b[:, None] * Kg)
        Ut = T @ (b[:, None] * V)
        U = Ut - W @ S
        Kh = (Gam[None, :] / gam) * K
        fw.append(dict(sl=sl, K=K, Q=Q, V=V, b=b, n=n, G=G, E=E, A=A, P=P, gam=gam, Gam=Gam,
                       T=T, Kg=Kg, Qg=Qg, W=W, U=U, Kh=Kh, S=S.copy(), ii=ii, jj=jj))
        S = Gam[:, None] * S + Kh.T @ U
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dg": np.zeros_like(g), "dbeta": np.zeros_like(beta)}
    # serial reverse pass over chunk-end cotangents
    dS = d_fin.copy()
    for f in reversed(fw):
        dO = d_o[f["sl"]]
        dSn = dS
        dU = f["P"].T @ dO + f["Kh"] @ dSn
        dS = f["Gam"][:, None] * dSn + f["Qg"].T @ dO - f["W"].T @ dU
        f["dSn"], f["dU"] = dSn, dU
    out["d_initial"] = dS
    # chunk-parallel gradients
    for f in fw:
        sl, K, Q, V, b, E, S = f["sl"], f["K"], f["Q"], f["V"], f["b"], f["E"], f["S"]
        ii, jj, T, U, dU, dSn = f["ii"], f["jj"], f["T"], f["U"], f["dU"], f["dSn"]
        dO = d_o[sl]
        dQg = dO @ S.T
        dP = (dO @ U.T) * (ii >= jj)
        dKh = U @ dSn.T
        dGam = (dSn * S).sum(1)
        dW = -dU @ S.T
        TdU, TdW = T.T @ dU, T.T @ dW
        dV = b[:, None] * TdU
        dKg = b[:, None] * TdW
        dbeta = (TdU * V).sum(1) + (TdW * f["Kg"]).sum(1)
        dT = dU @ (b[:, None] * V).T + dW @ (b[:, None] * f["Kg"]).T
        dZ = -T.T @ dT @ T.T
        dA = b[:, None] * dZ * (ii > jj)
        dbeta += (dZ * f["A"] * (ii > jj)).sum(1)
        a1 = np.einsum("ts,sc,tsc->tc", dA, K, E)      # sum_{s<t} dA_ts k_s e^{G_t - G_s}
        a2 = np.einsum("ts,tc,tsc->sc", dA, K, E)      # sum_{t>s} dA_ts k_t e^{G_t - G_s}
        p1 = np.einsum("ts,sc,tsc->tc", dP, K, E)      # sum_{s<=t} dP_ts k_s e^{G_t - G_s}
        p2 = np.einsum("ts,tc,tsc->sc", dP, Q, E)      # sum_{t>=s} dP_ts q_t e^{G_t - G_s}
        gam, Gam, Kh = f["gam"], f["Gam"], f["Kh"]
        dQ = p1 + dQg * gam
        dK = a1 + a2 + p2 + dKg * gam + dKh * (Gam[None, :] / gam)
        dG = K * a1 - K * a2 + Q * p1 - K * p2 + dQg * f["Qg"] + dKg * f["Kg"] - dKh * Kh
        dG[-1] += (dKh * Kh).sum(0) + dGam * Gam
        out["dq"][sl], out["dk"][sl], out["dv"][sl] = dQ, dK, dV
        out["dg"][sl] = np.cumsum(dG[::-1], axis=0)[::-1]
        out["dbeta"][sl] = dbeta
    return out


def read_golden(name):
    """Parse a fixture: header keys dk/dv/s0, then 'token <inputs> | <S_t> <o_t>'."""
    dk = dv = None
    s0 = None
    toks = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split(None, 1)
            if key == "dk":
                dk = int(rest)
            elif key == "dv":
                dv = int(rest)
            elif key == "s0":
                s0 = np.array([float(x) for x in rest.split()]).reshape(dk, dv)
            elif key == "token":
                lhs, rhs = rest.split("|")
                a = [float(x) for x in lhs.split()]
                e = [float(x) for x in rhs.split()]
                kk = a[0:dk]
                vv = a[dk:dk + dv]
                qq = a[dk + dv:2 * dk + dv]
                bb = a[2 * dk + dv]
                al = a[2 * dk + dv + 1:3 * dk + dv + 1]
                toks.append(dict(k=kk, v=vv, q=qq, beta=bb, alpha=al,
                                 S=np.array(e[:dk * dv]).reshape(dk, dv), o=np.array(e[dk * dv:])))
    return dk, dv, s0, toks


# ----------------------------------------------------------------------------
# Pins
# ----------------------------------------------------------------------------

def pin_identity_beta0(lib):
    x = rand_inputs([5, 0, 9], H=2, dk=6, dv=4, seed=1, s0_std=1.0)
    x["beta"][:] = 0.0
    x["g"][:] = 0.0
    r = _run(lib, x)
    assert np.array_equal(r["final_state"], x["s0"]), "beta=0, alpha=1 must leave S unchanged"
    for req in range(3):
        for t in range(x["cu"][req], x["cu"][req + 1]):
            for h in range(2):
                ref = x["s0"][req, h].T @ x["q"][t, h]
                np.testing.assert_allclose(r["o"][t, h], ref, rtol=0, atol=1e-13)


def pin_orthonormal_retrieval(lib):
    rng = _rng(2)
    dk, dv, n = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :n].T[:, None, :]                     # n orthonormal keys, H=1
    v = rng.standard_normal((n, 1, dv))
    x = dict(q=k.copy(), k=k, v=v, g=np.zeros((n, 1, dk)), beta=np.ones((n, 1)),
             cu=np.array([0, n], dtype=np.int64), s0=None)
    S = _run(lib, x)["final_state"][0, 0]
    for j in range(n):
        np.testing.assert_allclose(S.T @ k[j, 0], v[j, 0], rtol=0, atol=1e-12)


def pin_self_query(lib):
    x = rand_inputs([17], H=2, dk=8, dv=3, seed=3, s0_std=1.0)
    x["beta"][:] = 1.0
    x["q"] = x["k"].copy()
    r = _run(lib, x)
    np.testing.assert_allclose(r["o"], x["v"], rtol=0, atol=1e-12)


def pin_decay_closed_form(lib):
    x = rand_inputs([7, 11], H=3, dk=5, dv=4, seed=4, s0_std=1.0)
    x["beta"][:] = 0.0
    r = _run(lib, x)
    for req in range(2):
        lo, hi = x["cu"][req], x["cu"][req + 1]
        for h in range(3):
            G = np.cumsum(x["g"][lo:hi, h], axis=0)
            for i, t in enumerate(range(lo, hi)):
                St = np.exp(G[i])[:, None] * x["s0"][req, h]
                np.testing.assert_allclose(r["o"][t, h], St.T @ x["q"][t, h], rtol=1e-12,
                                           atol=1e-14)
            np.testing.assert_allclose(r["final_state"][req, h],
                                       np.exp(G[-1])[:, None] * x["s0"][req, h],
                                       rtol=1e-12, atol=1e-14)


def pin_golden_fixtures(lib):
    for name in ("scalar_d1.txt", "two_channel_dk2.txt"):
        dk, dv, s0, toks = read_golden(name)
        L = len(toks)
        q = np.array([t["q"] for t in toks])[:, None, :]
        k = np.array([t["k"] for t in toks])[:, None, :]
        v = np.array([t["v"] for t in toks])[:, None, :]
        g = np.log(np.array([t["alpha"] for t in toks]))[:, None, :]
        beta = np.array([t["beta"] for t in toks])[:, None]
        # states after each prefix come from snapshots at stride 1
        r = oracle.prefill(q, k, v, g, beta, np.array([0, L]), s0[None, None],
                           snapshot_stride=1, lib=lib)
        for i, t in enumerate(toks):
            np.testing.assert_allclose(r["snapshots"][i, 0], t["S"], rtol=0, atol=1e-12,
                                       err_msg=f"{name} token {i + 1} state")
            np.testing.assert_allclose(r["o"][i, 0], t["o"], rtol=0, atol=1e-12,
                                       err_msg=f"{name} token {i + 1} output")


def pin_brute_force(lib):
    cases = [([16], 1, 8, 8, -5.0), ([3, 16, 1], 2, 4, 6, -0.1), ([12, 5], 2, 7, 3, -1.0)]
    for seed, (lengths, H, dk, dv, gate_lo) in enumerate(cases):
        x = rand_inputs(lengths, H, dk, dv, seed=10 + seed, s0_std=0.5, gate_lo=gate_lo)
        stride = 4
        r = _run(lib, x, stride=stride)
        cs = r["cu_snapshots"]
        for req in range(len(lengths)):
            lo, hi = x["cu"][req], x["cu"][req + 1]
            for h in range(H):
                sl = slice(lo, hi)
                o, states = brute_force_chain(x["q"][sl, h], x["k"][sl, h], x["v"][sl, h],
                                              x["g"][sl, h], x["beta"][sl, h], x["s0"][req, h])
                np.testing.assert_allclose(r["o"][sl, h], o, rtol=0, atol=1e-13)
                fin = states[-1] if hi > lo else x["s0"][req, h]
                np.testing.assert_allclose(r["final_state"][req, h], fin, rtol=0, atol=1e-13)
                for j in range(1, (hi - lo) // stride + 1):
                    np.testing.assert_allclose(r["snapshots"][cs[req] + j - 1, h],
                                               states[j * stride - 1], rtol=0, atol=1e-13)


def pin_chunked_form(lib):
    for gate_lo in (-5.0, -0.05):   # strong decay (exponent range) and weak (long range)
        _chunked_case(lib, gate_lo)


def _chunked_case(lib, gate_lo):
    L, H, dk, dv = 150, 2, 8, 6
    x = rand_inputs([L], H, dk, dv, seed=21, s0_std=0.3, gate_lo=gate_lo)
    r = _run(lib, x)
    for C in (1, 16, 64, L):
        for h in range(H):
            O, S = chunked_chain(x["q"][:, h], x["k"][:, h], x["v"][:, h], x["g"][:, h],
                                 x["beta"][:, h], x["s0"][0, h], C)
            np.testing.assert_allclose(O, r["o"][:, h], rtol=0, atol=1e-10,
                                       err_msg=f"chunked C={C}")
            np.testing.assert_allclose(S, r["final_state"][0, h], rtol=0, atol=1e-10)


def pin_split_combine(lib):
    # weak decay, so the transition M stays far from zero and its errors show
    L, H, dk, dv, seg = 96, 2, 6, 5, 24
    x = rand_inputs([L], H, dk, dv, seed=31, s0_std=0.7, gate_lo=-0.05)
    full = _run(lib, x, stride=seg)
    seg_cu = np.arange(0, L + 1, seg)
    s_loc, m = oracle.chunk_local_state(x["k"], x["v"], x["g"], x["beta"], seg_cu, lib=lib)
    s_in, s_fin = oracle.state_combine(s_loc, m, x["s0"][0], lib=lib)
    np.testing.assert_allclose(s_fin, full["final_state"][0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_in[0], x["s0"][0], rtol=0, atol=0)
    for s in range(1, len(seg_cu) - 1):
        np.testing.assert_allclose(s_in[s], full["snapshots"][s - 1], rtol=0, atol=1e-12)
    # M alone: brute-force product of the dense transitions of segment 1, head 1
    lo, hi = seg_cu[1], seg_cu[2]
    Mref = np.eye(dk)
    for t in range(lo, hi):
        A = (np.eye(dk) - x["beta"][t, 1] * np.outer(x["k"][t, 1], x["k"][t, 1])) \
            @ np.diag(np.exp(x["g"][t, 1]))
        Mref = A @ Mref
    np.testing.assert_allclose(m[1, 1], Mref, rtol=0, atol=1e-13)


def pin_snapshot_tagging(lib):
    """beta=1, alpha=1, one-hot keys: the write at position p replaces row p mod dk
    with v_p, so each row of a snapshot names the last position written into it."""
    dk, dv, stride = 8, 1, 4
    lengths = [19, 8, 3]
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    k = np.zeros((T, 1, dk))
    v = np.zeros((T, 1, dv))
    for r_ in range(len(lengths)):
        for p in range(lengths[r_]):
            k[cu[r_] + p, 0, p % dk] = 1.0
            v[cu[r_] + p, 0, 0] = 100 * (r_ + 1) + p + 1   # encodes request and position
    x = dict(q=k.copy(), k=k, v=v, g=np.zeros((T, 1, dk)), beta=np.ones((T, 1)), cu=cu, s0=None)
    r = _run(lib, x, stride=stride)
    assert r["snapshots"].shape[0] == sum(L // stride for L in lengths)
    idx = 0
    for r_, L in enumerate(lengths):
        for j in range(1, L // stride + 1):
            n = j * stride                      # tokens consumed
            exp_ = np.zeros(dk)
            for p in range(n):
                exp_[p % dk] = 100 * (r_ + 1) + p + 1
            assert np.array_equal(r["snapshots"][idx, 0, :, 0], exp_), (r_, j)
            idx += 1


def pin_contraction_bound(lib):
    x = rand_inputs([40], H=1, dk=6, dv=4, seed=41, s0_std=2.0)
    state = np.ascontiguousarray(x["s0"].copy())
    for t in range(40):
        prev = np.linalg.norm(state[0, 0], 2)
        oracle.decode_step(x["q"][t:t + 1], x["k"][t:t + 1], x["v"][t:t + 1],
                           x["g"][t:t + 1], x["beta"][t:t + 1], state, lib=lib)
        bound = prev + x["beta"][t, 0] * np.linalg.norm(x["k"][t, 0]) * np.linalg.norm(x["v"][t, 0])
        assert np.linalg.norm(state[0, 0], 2) <= bound * (1 + 1e-12)


def pin_resume(lib):
    L, stride = 45, 8
    x = rand_inputs([L], H=2, dk=5, dv=5, seed=51, s0_std=0.4, gate_lo=-0.1)
    full = _run(lib, x, stride=stride)
    for j in (1, 3, 5):
        cut = j * stride
        y = {kk: (vv[cut:] if kk in ("q", "k", "v", "g", "beta") else vv) for kk, vv in x.items()}
        y["cu"] = np.array([0, L - cut], dtype=np.int64)
        y["s0"] = full["snapshots"][j - 1][None]
        part = _run(lib, y)
        np.testing.assert_allclose(part["o"], full["o"][cut:], rtol=0, atol=1e-12)
        np.testing.assert_allclose(part["final_state"], full["final_state"], rtol=0, atol=1e-12)


def pin_decode_matches_prefill(lib):
    L, N, H, dk, dv = 12, 3, 2, 6, 5
    x = rand_inputs([L] * N, H, dk, dv, seed=61, s0_std=0.5, gate_lo=-0.2)
    full = _run(lib, x)
    state = np.ascontiguousarray(x["s0"].copy())
    for t in range(L):
        rows = [x["cu"][n] + t for n in range(N)]
        o = oracle.decode_step(x["q"][rows], x["k"][rows], x["v"][rows], x["g"][rows],
                               x["beta"][rows], state, lib=lib)
        np.testing.assert_allclose(o, full["o"][rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(state, full["final_state"], rtol=0, atol=1e-12)


def pin_decode_slots(lib):
    x = rand_inputs([1, 1, 1], H=2, dk=4, dv=3, seed=71)
    rng = _rng(72)
    pool = rng.standard_normal((5, 2, 4, 3))
    state = np.ascontiguousarray(pool.copy())
    slot = np.array([4, 0, 2], dtype=np.int64)
    oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state, slot=slot, lib=lib)
    for s in (1, 3):
        assert np.array_equal(state[s], pool[s]), "untouched slots must not change"
    for n, s in enumerate(slot):
        _, states = brute_force_chain(x["q"][n:n + 1, 0], x["k"][n:n + 1, 0], x["v"][n:n + 1, 0],
                                      x["g"][n:n + 1, 0], x["beta"][n:n + 1, 0], pool[s, 0])
        np.testing.assert_allclose(state[s, 0], states[-1], rtol=0, atol=1e-13)


def pin_varlen_isolation(lib):
    lengths = [13, 0, 30, 7]
    x = rand_inputs(lengths, H=2, dk=5, dv=4, seed=81, s0_std=0.5, gate_lo=-0.2)
    packed = _run(lib, x, stride=4)
    for r_ in range(len(lengths)):
        lo, hi = x["cu"][r_], x["cu"][r_ + 1]
        y = {kk: (vv[lo:hi] if kk in ("q", "k", "v", "g", "beta") else vv) for kk, vv in x.items()}
        y["cu"] = np.array([0, hi - lo], dtype=np.int64)
        y["s0"] = x["s0"][r_:r_ + 1]
        alone = _run(lib, y, stride=4)
        assert np.array_equal(alone["o"], packed["o"][lo:hi])
        assert np.array_equal(alone["final_state"][0], packed["final_state"][r_])
        cs = packed["cu_snapshots"]
        assert np.array_equal(alone["snapshots"], packed["snapshots"][cs[r_]:cs[r_ + 1]])


# ----------------------------------------------------------------------------
# Backward (vector-Jacobian product of the prefill map)
# ----------------------------------------------------------------------------

_GRAD_OF = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "s0": "d_initial"}


def _loss(lib, x, d_o, d_fin):
    r = _run(lib, x)
    return float((r["o"] * d_o).sum() + (r["final_state"] * d_fin).sum())


def _backward(lib, x, d_o, d_fin):
    return oracle.prefill_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu"], x["s0"],
                                   d_o, d_fin, n_threads=2, lib=lib)


def _fd_check(lib, x, d_o, d_fin, n_sample=None, seed=0, h=1e-6, tol=1e-6):
    """Central differences of the forward oracle's scalar loss against the
    backward's gradients, element by element (all, or n_sample per input)."""
    grads = _backward(lib, x, d_o, d_fin)
    rng = _rng(seed)
    for name, gname in _GRAD_OF.items():
        a = x[name]
        idx = list(np.ndindex(a.shape))
        if n_sample is not None:
            idx = [idx[i] for i in rng.choice(len(idx), size=min(n_sample, len(idx)), replace=False)]
        scale = max(np.abs(grads[gname]).max(), 1e-12)
        for ix in idx:
            keep = a[ix]
            a[ix] = keep + h
            lp = _loss(lib, x, d_o, d_fin)
            a[ix] = keep - h
            lm = _loss(lib, x, d_o, d_fin)
            a[ix] = keep
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grads[gname][ix]) <= tol * scale, (name, ix, fd, grads[gname][ix])


def pin_backward_finite_differences(lib):
    """Every gradient element of a small varlen case (two requests, an initial
    state, random cotangents) equals the central difference of the forward."""
    x = rand_inputs([5, 9], H=2, dk=3, dv=4, seed=71, gate_lo=-1.0, s0_std=1.0)
    rng = _rng(72)
    d_o = rng.standard_normal(x["v"].shape)
    d_fin = rng.standard_normal(x["s0"].shape)
    _fd_check(lib, x, d_o, d_fin)


def pin_backward_across_blocks(lib):
    """A 150-token chain crosses the backward's 64-token recompute blocks twice;
    sampled elements of every gradient still match central differences."""
    x = rand_inputs([150], H=1, dk=3, dv=2, seed=73, gate_lo=-0.5, s0_std=1.0)
    rng = _rng(74)
    d_o = rng.standard_normal(x["v"].shape)
    d_fin = rng.standard_normal(x["s0"].shape)
    _fd_check(lib, x, d_o, d_fin, n_sample=40, seed=75)


def pin_backward_beta0_closed_form(lib):
    """beta = 0 and dO = 0: S_L = Diag(gamma_L) S_0 with gamma_L = exp(sum_t g_t), so
    dS_0 = Diag(gamma_L) dS_L, dg_t,i = gamma_L,i sum_j dS_L,ij S_0,ij for every t,
    dq = dk = dv = 0, and dbeta_t = k_t^T Diag(gamma_L / gamma_t) dS_L
    (v_t - (Diag(gamma_t) S_0)^T k_t) with gamma_t the decay over tokens 1..t."""
    x = rand_inputs([11], H=1, dk=4, dv=3, seed=76, s0_std=1.0)
    x["beta"][:] = 0.0
    rng = _rng(77)
    d_fin = rng.standard_normal(x["s0"].shape)
    r = _backward(lib, x, None, d_fin)
    g = x["g"][:, 0]
    S0, dF = x["s0"][0, 0], d_fin[0, 0]
    gam_L = np.exp(g.sum(0))
    np.testing.assert_allclose(r["d_initial"][0, 0], gam_L[:, None] * dF, rtol=1e-12, atol=1e-14)
    for name in ("dq", "dk", "dv"):
        assert np.array_equal(r[name], np.zeros_like(r[name])), name
    row = gam_L * (dF * S0).sum(1)
    for t in range(11):
        np.testing.assert_allclose(r["dg"][t, 0], row, rtol=1e-12, atol=1e-14)
        gam_t = np.exp(g[:t + 1].sum(0))
        kt = x["k"][t, 0]
        ref = kt @ ((gam_L / gam_t)[:, None] * dF) @ (x["v"][t, 0] - (gam_t[:, None] * S0).T @ kt)
        np.testing.assert_allclose(r["dbeta"][t, 0], ref, rtol=1e-10, atol=1e-13)


def pin_backward_dq_is_state_times_cotangent(lib):
    """o_t = S_t^T q_t makes dq_t = S_t dO_t exactly; S_t is read from the forward
    oracle's snapshots at stride 1 (dS_L = 0)."""
    x = rand_inputs([7, 12], H=2, dk=5, dv=3, seed=78, s0_std=0.5)
    rng = _rng(79)
    d_o = rng.standard_normal(x["v"].shape)
    r = _backward(lib, x, d_o, None)
    f = _run(lib, x, stride=1)
    for t in range(19):
        for h in range(2):
            np.testing.assert_allclose(r["dq"][t, h], f["snapshots"][t, h] @ d_o[t, h],
                                       rtol=1e-12, atol=1e-13)


def pin_backward_chunked_form(lib):
    """The oracle's backward equals the reverse mode of the chunked form at chunk
    sizes 1, 16, 64 and the whole sequence, strong and weak decay."""
    for gate_lo in (-5.0, -0.05):
        L, H, dk, dv = 150, 2, 8, 6
        x = rand_inputs([L], H, dk, dv, seed=81, s0_std=0.3, gate_lo=gate_lo)
        rng = _rng(82)
        d_o = rng.standard_normal(x["v"].shape)
        d_fin = rng.standard_normal(x["s0"].shape)
        r = _backward(lib, x, d_o, d_fin)
        for C in (1, 16, 64, L):
            for h in range(H):
                c = chunked_backward_chain(x["q"][:, h], x["k"][:, h], x["v"][:, h],
                                           x["g"][:, h], x["beta"][:, h], x["s0"][0, h],
                                           d_o[:, h], d_fin[0, h], C)
                for name in ("dq", "dk", "dv", "dg", "dbeta"):
                    ref = r[name][:, h]
                    np.testing.assert_allclose(c[name], ref, rtol=0,
                                               atol=1e-9 * max(1.0, np.abs(ref).max()),
                                               err_msg=f"{name} C={C} gate_lo={gate_lo}")
                np.testing.assert_allclose(c["d_initial"], r["d_initial"][0, h], rtol=0,
                                           atol=1e-9 * max(1.0, np.abs(r["d_initial"]).max()))


# ----------------------------------------------------------------------------
# Fused gate activation: log(alpha) = -5 sigmoid(x) of bf16 logits x (the
# lower-bounded decay, CSDN post on the Kimi K3 technical report, section 一.1)
# ----------------------------------------------------------------------------

def pin_gate_logit_map(lib):
    """Values fixed by the sigmoid itself: g(0) = -2.5, g(x) + g(-x) = -5 (as
    sigmoid(x) + sigmoid(-x) = 1), g in [-5, 0] and decreasing, the limits -0 and
    -5 at the ends of the range, and the slope equal to central differences."""
    del lib
    assert oracle.gate_from_logits(np.array([0.0]))[0] == -2.5
    x = np.linspace(-30.0, 30.0, 601)
    gx = oracle.gate_from_logits(x)
    np.testing.assert_allclose(gx + oracle.gate_from_logits(-x), -5.0, rtol=0, atol=1e-14)
    assert np.all(gx <= 0.0) and np.all(gx >= -5.0) and np.all(np.diff(gx) < 0.0)
    ends = oracle.gate_from_logits(np.array([-800.0, 800.0]))
    assert ends[0] == 0.0 and ends[1] == -5.0
    h = 1e-5
    fd = (oracle.gate_from_logits(x + h) - oracle.gate_from_logits(x - h)) / (2 * h)
    np.testing.assert_allclose(oracle.gate_logit_slope(x), fd, rtol=0, atol=1e-9)


def pin_gate_logit_decay(lib):
    """beta = 0 and every logit 0: alpha = exp(-2.5) on every channel, so
    S_t = exp(-2.5 t) S_0 and o_t = S_t^T q_t (the decay closed form)."""
    x = rand_inputs([6, 9], H=2, dk=4, dv=3, seed=83, s0_std=1.0)
    x["beta"][:] = 0.0
    logits = np.zeros_like(x["g"])
    r = oracle.prefill(x["q"], x["k"], x["v"], None, x["beta"], x["cu"], x["s0"],
                       n_threads=2, lib=lib, g_logits=logits)
    for req in range(2):
        lo, hi = x["cu"][req], x["cu"][req + 1]
        for h in range(2):
            for i, t in enumerate(range(lo, hi)):
                St = np.exp(-2.5 * (i + 1)) * x["s0"][req, h]
                np.testing.assert_allclose(r["o"][t, h], St.T @ x["q"][t, h], rtol=1e-12,
                                           atol=1e-15)
            np.testing.assert_allclose(r["final_state"][req, h],
                                       np.exp(-2.5 * (hi - lo)) * x["s0"][req, h],
                                       rtol=1e-12, atol=1e-15)


def pin_gate_logit_backward(lib):
    """The gradient the backward returns for logits equals central differences of
    the forward loss taken in the logits themselves."""
    x = rand_inputs([5, 8], H=2, dk=3, dv=2, seed=84, s0_std=1.0)
    rng = _rng(85)
    logits = rng.standard_normal(x["g"].shape)
    d_o = rng.standard_normal(x["v"].shape)
    d_fin = rng.standard_normal(x["s0"].shape)

    def loss(lg):
        r = oracle.prefill(x["q"], x["k"], x["v"], None, x["beta"], x["cu"], x["s0"],
                           n_threads=2, lib=lib, g_logits=lg)
        return float((r["o"] * d_o).sum() + (r["final_state"] * d_fin).sum())

    grads = oracle.prefill_backward(x["q"], x["k"], x["v"], None, x["beta"], x["cu"], x["s0"],
                                    d_o, d_fin, n_threads=2, lib=lib, g_logits=logits)
    scale = max(np.abs(grads["dg"]).max(), 1e-12)
    h = 1e-6
    for ix in np.ndindex(logits.shape):
        keep = logits[ix]
        logits[ix] = keep + h
        lp = loss(logits)
        logits[ix] = keep - h
        lm = loss(logits)
        logits[ix] = keep
        fd = (lp - lm) / (2 * h)
        assert abs(fd - grads["dg"][ix]) <= 1e-6 * scale, (ix, fd, grads["dg"][ix])


ALL_PINS = [pin_identity_beta0, pin_orthonormal_retrieval, pin_self_query,
            pin_decay_closed_form, pin_golden_fixtures, pin_brute_force, pin_chunked_form,
            pin_split_combine, pin_snapshot_tagging, pin_contraction_bound, pin_resume,
            pin_decode_matches_prefill, pin_decode_slots, pin_varlen_isolation,
            pin_backward_finite_differences, pin_backward_across_blocks,
            pin_backward_beta0_closed_form, pin_backward_dq_is_state_times_cotangent,
            pin_backward_chunked_form, pin_gate_logit_map, pin_gate_logit_decay,
            pin_gate_logit_backward]
