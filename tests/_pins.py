"""Independent evaluations used to pin the oracle (CPU, numpy, fp64).

None of these reuse the oracle's recurrences: they evaluate the defining sums
directly (O(T^2) or O(T^2 K V)), or use a different algorithm (chunked
evaluation, finite differences), so a slip in the oracle shows up as a
mismatch here.
"""

import numpy as np


def rel_err(x, ref, floor=0.0):
    """max_i |x_i - ref_i| / max(|ref_i|, rms(ref), floor).

    The denominator is floored at the RMS of the reference tensor so that
    entries near zero (cancelling sums) do not dominate, and at `floor` for
    references that are zero up to round-off.
    """
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    floor = max(float(np.sqrt(np.mean(ref ** 2))), floor)
    den = np.maximum(np.abs(ref), floor)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(x - ref) / den))


def wkv4_direct_sum(w, u, k, v):
    """RWKV-4 y_t from the definition, one t at a time.

    Token t sees exponents -(t-1-i) w + k_i for each past token i < t and
    u + k_t for itself; y_t is the softmax of those exponents applied to v.
    """
    w, u, k, v = (np.asarray(a, dtype=np.float64) for a in (w, u, k, v))
    B, T, C = k.shape
    y = np.empty_like(k)
    for t in range(T):
        i = np.arange(t)
        # [B, t+1, C] exponents
        past = -(t - 1 - i)[None, :, None] * w[None, None, :] + k[:, :t, :]
        cur = (u[None, :] + k[:, t, :])[:, None, :]
        ex = np.concatenate([past, cur], axis=1)
        vals = np.concatenate([v[:, :t, :], v[:, t:t + 1, :]], axis=1)
        m = ex.max(axis=1, keepdims=True)
        p = np.exp(ex - m)
        y[:, t, :] = (p * vals).sum(axis=1) / p.sum(axis=1)
    return y


def wkv6_direct_sum(r, k, v, w, u, K):
    """RWKV-6 o_t from the unrolled state, per head:

    o_t[j] = sum_i r_t[i] ( sum_{s<t} prod_{tau=s+1}^{t-1} w_tau[i] k_s[i] v_s[j]
                            + u[i] k_t[i] v_t[j] )
    """
    r, k, v, w = (np.asarray(a, dtype=np.float64) for a in (r, k, v, w))
    u = np.asarray(u, dtype=np.float64).reshape(-1)
    B, T, HK = r.shape
    H = HK // K
    o = np.zeros_like(r)
    for b in range(B):
        for h in range(H):
            sl = slice(h * K, (h + 1) * K)
            R, Kk, V, W = r[b, :, sl], k[b, :, sl], v[b, :, sl], w[b, :, sl]
            for t in range(T):
                acc = np.zeros(K)
                for s in range(t):
                    dec = np.prod(W[s + 1:t], axis=0) if t - 1 >= s + 1 else np.ones(K)
                    acc += (R[t] * dec * Kk[s]).sum() * V[s]
                acc += (R[t] * u[sl] * Kk[t]).sum() * V[t]
                o[b, t, sl] = acc
    return o


def wkv6_chunked(r, k, v, w, u, K, L, init_state=None):
    """RWKV-6 forward by the chunked form (chunk length L), in fp64.

    Per chunk with lam_j = sum_{tau<=j} ln w_tau (lam_{-1} = 0):
      o_j  = (r_j * e^{lam_{j-1}}) S_in
             + sum_{s<j} [sum_i r_j[i] e^{lam_{j-1}[i]-lam_s[i]} k_s[i]] v_s
             + [sum_i r_j[i] u[i] k_j[i]] v_j
      S_out = diag(e^{lam_{L-1}}) S_in + sum_s (k_s * e^{lam_{L-1}-lam_s})^T v_s
    Returns (o, final_state [B, H, K, K]).
    """
    r, k, v, w = (np.asarray(a, dtype=np.float64) for a in (r, k, v, w))
    u = np.asarray(u, dtype=np.float64).reshape(-1)
    B, T, HK = r.shape
    H = HK // K
    o = np.zeros_like(r)
    fs = np.zeros((B, H, K, K))
    for b in range(B):
        for h in range(H):
            sl = slice(h * K, (h + 1) * K)
            S = np.zeros((K, K)) if init_state is None else np.array(init_state[b, h], dtype=np.float64)
            for t0 in range(0, T, L):
                t1 = min(T, t0 + L)
                R, Kk, V, W = r[b, t0:t1, sl], k[b, t0:t1, sl], v[b, t0:t1, sl], w[b, t0:t1, sl]
                n = t1 - t0
                lam = np.cumsum(np.log(W), axis=0)                     # lam_j
                lam_prev = np.vstack([np.zeros((1, K)), lam[:-1]])    # lam_{j-1}
                out = (R * np.exp(lam_prev)) @ S
                A = np.zeros((n, n))
                for j in range(n):
                    for s in range(j):
                        A[j, s] = (R[j] * np.exp(lam_prev[j] - lam[s]) * Kk[s]).sum()
                    A[j, j] = (R[j] * u[sl] * Kk[j]).sum()
                out += A @ V
                o[b, t0:t1, sl] = out
                S = np.exp(lam[-1])[:, None] * S + (Kk * np.exp(lam[-1][None, :] - lam)).T @ V
            fs[b, h] = S
    return o, fs


def wkv4_fd_grads(fwd, w, u, k, v, gy):
    """Central finite differences of L = sum(gy * fwd(w, u, k, v)).

    Step h = 1e-5 * max(1, |x|). Returns (gk, gv, gw, gu).
    """
    w, u, k, v = (np.array(a, dtype=np.float64) for a in (w, u, k, v))

    def loss():
        return float((fwd(w, u, k, v) * gy).sum())

    def fd(arr, idx):
        x0 = arr[idx]
        h = 1e-5 * max(1.0, abs(x0))
        arr[idx] = x0 + h
        lp = loss()
        arr[idx] = x0 - h
        lm = loss()
        arr[idx] = x0
        return (lp - lm) / (2 * h)

    gk = np.zeros_like(k)
    gv = np.zeros_like(v)
    for idx in np.ndindex(*k.shape):
        gk[idx] = fd(k, idx)
        gv[idx] = fd(v, idx)
    gw = np.array([fd(w, (c,)) for c in range(w.shape[0])])
    gu = np.array([fd(u, (c,)) for c in range(u.shape[0])])
    return gk, gv, gw, gu


def wkv6_fd_grads(fwd, r, k, v, w, u, dout, init_state=None, g_final=None):
    """Central finite differences of L = sum(o * dout) + sum(fs * g_final)
    for (o, fs) = fwd(r, k, v, w, u, init_state=...). Step 1e-5 * max(1, |x|).
    Returns (gr, gk, gv, gw, gu [flat H*K], g_init or None)."""
    arrs = {n: np.array(a, dtype=np.float64) for n, a in
            (("r", r), ("k", k), ("v", v), ("w", w), ("u", u))}
    s0 = None if init_state is None else np.array(init_state, dtype=np.float64)

    def loss():
        kw = {} if s0 is None else {"init_state": s0}
        o, fs = fwd(arrs["r"], arrs["k"], arrs["v"], arrs["w"], arrs["u"], **kw)
        L = float((o * dout).sum())
        if g_final is not None:
            L += float((fs * g_final).sum())
        return L

    def fd(arr, idx):
        x0 = arr[idx]
        h = 1e-5 * max(1.0, abs(x0))
        arr[idx] = x0 + h
        lp = loss()
        arr[idx] = x0 - h
        lm = loss()
        arr[idx] = x0
        return (lp - lm) / (2 * h)

    out = []
    for n in ("r", "k", "v", "w", "u"):
        a = arrs[n]
        g = np.zeros_like(a)
        for idx in np.ndindex(*a.shape):
            g[idx] = fd(a, idx)
        out.append(g.reshape(-1) if n == "u" else g)
    gi = None
    if s0 is not None:
        gi = np.zeros_like(s0)
        for idx in np.ndindex(*s0.shape):
            gi[idx] = fd(s0, idx)
    return tuple(out) + (gi,)
